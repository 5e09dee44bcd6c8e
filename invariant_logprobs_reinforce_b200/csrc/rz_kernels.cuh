// rz_kernels.cuh -- the epilogues that turn the tensor-core engine into the four
// contractions of the path, and the SIMT kernels around them.
//
//   EpiLse       fused LM head + online log-sum-exp + gather (forward; logits stay on chip)
//   merge_lse    fixed-order merge of the per-segment (max, sum) pairs -> lse, lp
//   response_coef / token_kappa / loss_final
//                group-mean advantage, unclipped ratio, per-response token mean
//   EpiDz        recompute a logit tile, dZ = kappa (onehot - softmax) -> bf16
//   EpiStoreBf16 dH = dZ W tile store
//   EpiAccF32    dW (+)= dZ^T H tile read-modify-write, chunks in fixed order
//
// Definitions follow "vLLM says aligned kernels make asynchronous RL stable at lag 64"
// (ainewsbites.com), section "REINFORCE Zero removes the mismatch first"; the fixed
// orders follow "vLLM Train-Inference Consistency Release Notes" (agentlenshq.com),
// section "Achieving Bitwise Consistency" (kernel determinism, batch independence).
#pragma once

#include <cuda_bf16.h>

#include "rz_gemm.cuh"

namespace rz {

// Vocabulary segment of the forward: 8 tiles of 256 columns.  A function of nothing:
// the segment grid over [0, V) is fixed, so every row sees the same reduction order
// whatever the number of rows in the call.
constexpr int kSegTiles = 8;
constexpr int kSegWidth = kSegTiles * BN;  // 2048 vocabulary columns

// Backward chunk: tokens whose dZ rows are materialised at once (a fixed constant, so
// the order in which token contributions reach dW never depends on n_tok).
constexpr int kChunkTokens = 16384;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// ------------------------------------------------------------------------ forward

struct EpiLse {
  const int32_t* ids;
  int64_t n;        // rows
  int V;
  float* part_m;    // [S][n] running max of the segment
  float* part_s;    // [S][n] sum of exp(z - max) over the segment
  float* zy;        // [n]    logit of the sampled token

  struct State {
    float m, s;
    int y;
    int64_t row;
  };

  __device__ __forceinline__ void begin_unit(State& st, int mb, int, int r) const {
    st.row = static_cast<int64_t>(mb) * BM + r;
    st.y = st.row < n ? __ldg(ids + st.row) : -1;
    st.m = -INFINITY;
    st.s = 0.0f;
  }

  __device__ __forceinline__ void tile(State& st, uint32_t taddr, int, int nt, int) const {
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int col0 = nt * BN + c * 32;
      if (col0 >= V) break;  // uniform across the warp
      float v[32];
      __syncwarp();  // the TMEM load is warp-collective: reconverge first
      tmem_ld_32cols(taddr + c * 32, v);
      if (col0 + 32 > V) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j >= V) v[j] = -INFINITY;
      }
      const unsigned off = static_cast<unsigned>(st.y - col0);
      if (off < 32u) {
        float z = v[0];
#pragma unroll
        for (int j = 1; j < 32; ++j) z = (static_cast<unsigned>(j) == off) ? v[j] : z;
        if (st.row < n) zy[st.row] = z;
      }
      float cmax = v[0];
#pragma unroll
      for (int j = 1; j < 32; ++j) cmax = fmaxf(cmax, v[j]);
      const float m_new = fmaxf(st.m, cmax);
      // exp(v - m) as 2^((v - m) log2 e): the maximum contributes exactly 1
      float acc = st.s * ex2_approx((st.m - m_new) * kLog2e);
#pragma unroll
      for (int j = 0; j < 32; ++j) acc += ex2_approx((v[j] - m_new) * kLog2e);
      st.s = acc;
      st.m = m_new;
    }
  }

  __device__ __forceinline__ void end_unit(const State& st, int, int nu, int) const {
    if (st.row < n) {
      part_m[static_cast<int64_t>(nu) * n + st.row] = st.m;
      part_s[static_cast<int64_t>(nu) * n + st.row] = st.s;
    }
  }
};

// lse = M + log(sum_s s_s 2^{(m_s - M) log2 e}), segments merged in order s = 0..S-1.
__global__ void merge_lse_kernel(const float* __restrict__ part_m, const float* __restrict__ part_s,
                                 const float* __restrict__ zy, const int32_t* __restrict__ ids, int64_t n, int V,
                                 int S, float* __restrict__ lp, float* __restrict__ lse_out, int* status) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n) return;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, part_m[static_cast<int64_t>(s) * n + t]);
  float sum = 0.0f;
  for (int s = 0; s < S; ++s)
    sum += part_s[static_cast<int64_t>(s) * n + t] * ex2_approx((part_m[static_cast<int64_t>(s) * n + t] - M) * kLog2e);
  const float l = M + logf(sum);
  const int y = ids[t];
  if (y < 0 || y >= V) {
    atomicOr(status, kDevBadTokenId);
    lp[t] = __int_as_float(0x7fc00000);
  } else {
    lp[t] = zy[t] - l;
  }
  if (lse_out != nullptr) lse_out[t] = l;
}

// ------------------------------------------------------------------------ loss stage

// One block.  Checks the segments and groups, forms each group's reward sum in
// response-index order (fp64), and the per-response coefficient  coef_i = -A_i / (N L_i).
// When the group ids are non-decreasing (groups are contiguous runs, the usual layout),
// the first response of each run sums its run: O(R).  Otherwise every group scans all
// responses: O(R G).  Both add the same rewards in the same (index) order, so both give
// the same bits.
__global__ void __launch_bounds__(1024)
    response_coef_kernel(const float* __restrict__ rewards, const int64_t* __restrict__ off,
                         const int32_t* __restrict__ gid, int R, int G, int64_t n, double* __restrict__ gsum,
                         int* __restrict__ gcnt, float* __restrict__ coef, int* status) {
  int bad = 0;
  int sorted = 1;
  if (threadIdx.x == 0 && (off[0] != 0 || off[R] != n)) bad |= kDevBadSegments;
  for (int i = threadIdx.x; i < R; i += blockDim.x) {
    if (off[i + 1] <= off[i]) bad |= kDevBadSegments;
    const int g = gid[i];
    if (g < 0 || g >= G) bad |= kDevBadGroupId;
    if (i + 1 < R && gid[i + 1] < g) sorted = 0;
  }
  if (bad) atomicOr(status, bad);
  sorted = __syncthreads_and(sorted);
  if (sorted) {
    for (int i = threadIdx.x; i < R; i += blockDim.x) {
      const int g = gid[i];
      if ((i > 0 && gid[i - 1] == g) || g < 0 || g >= G) continue;  // not the start of a valid run
      double s = 0.0;
      int c = 0;
      for (int j = i; j < R && gid[j] == g; ++j) {
        s += static_cast<double>(rewards[j]);
        ++c;
      }
      gsum[g] = s;
      gcnt[g] = c;
    }
  } else {
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
      double s = 0.0;
      int c = 0;
      for (int i = 0; i < R; ++i) {
        if (__ldg(gid + i) == g) {
          s += static_cast<double>(__ldg(rewards + i));
          ++c;
        }
      }
      gsum[g] = s;
      gcnt[g] = c;
    }
  }
  __syncthreads();
  const double N = static_cast<double>(R);
  for (int i = threadIdx.x; i < R; i += blockDim.x) {
    const int g = gid[i];
    const int64_t L = off[i + 1] - off[i];
    if (g < 0 || g >= G || L <= 0) {
      coef[i] = __int_as_float(0x7fc00000);
    } else {
      const double A = static_cast<double>(rewards[i]) - gsum[g] / static_cast<double>(gcnt[g]);
      coef[i] = static_cast<float>(-A / (N * static_cast<double>(L)));
    }
  }
}

constexpr int kKappaThreads = 256;
constexpr int kKappaIters = 4;                                    // float4 groups per thread
constexpr int kKappaBlockTokens = kKappaThreads * 4 * kKappaIters;  // 4096 tokens per block
constexpr int kKappaStagedOffsets = 256;                          // responses staged per block

// response owning token t: the largest i with off[i] <= t (clamped to [0, R-1])
__device__ __forceinline__ int find_response(const int64_t* __restrict__ off, int R, int64_t t) {
  int lo = 0, hi = R - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(off + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// kappa_t = coef_i * exp(lp_t - lp_rollout_t) (ratio unclipped) for 4096 tokens per block;
// per-block partial sums of kappa in fp64 with a fixed reduction order.  The segment
// offsets a block touches are staged in shared memory once per block.
__global__ void __launch_bounds__(kKappaThreads)
    token_kappa_kernel(const float* __restrict__ lp, const float* __restrict__ lp_roll,
                       const int64_t* __restrict__ off, int R, const float* __restrict__ coef, int64_t n,
                       int vec_ok, float* __restrict__ kappa, float* __restrict__ w_out,
                       double* __restrict__ block_sums) {
  __shared__ int64_t s_off[kKappaStagedOffsets + 1];
  __shared__ int s_first, s_count;
  __shared__ double warp_sums[kKappaThreads / 32];
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * kKappaBlockTokens;
  const int64_t b1 = min(n, b0 + kKappaBlockTokens);
  if (threadIdx.x == 0) {
    const int i0 = find_response(off, R, b0);
    const int i1 = find_response(off, R, b1 - 1);
    s_first = i0;
    s_count = i1 - i0 + 1;
  }
  __syncthreads();
  const int i0 = s_first;
  const int cnt = s_count;
  const bool staged = cnt >= 1 && cnt <= kKappaStagedOffsets;
  if (staged)
    for (int k = threadIdx.x; k <= cnt; k += kKappaThreads) s_off[k] = off[i0 + k];
  __syncthreads();

  // offset of response i+1, from shared memory when staged (past the staged range, which
  // only malformed offsets can reach, the walk stops)
  auto next_off = [&](int i) -> int64_t {
    if (!staged) return __ldg(off + i + 1);
    return (i + 1 - i0) <= cnt ? s_off[i + 1 - i0] : INT64_MAX;
  };
  auto locate = [&](int64_t t) -> int {
    if (!staged) return find_response(off, R, t);
    int lo = 0, hi = cnt - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return i0 + lo;
  };

  double local = 0.0;
#pragma unroll 1
  for (int it = 0; it < kKappaIters; ++it) {
    const int64_t t0 = b0 + static_cast<int64_t>(it) * (kKappaThreads * 4) + threadIdx.x * 4;
    if (t0 >= b1) break;
    int i = locate(t0);
    if (vec_ok && t0 + 4 <= n) {
      const float4 a = *reinterpret_cast<const float4*>(lp + t0);
      const float4 b = *reinterpret_cast<const float4*>(lp_roll + t0);
      const float la[4] = {a.x, a.y, a.z, a.w};
      const float lb[4] = {b.x, b.y, b.z, b.w};
      float w[4], k[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        while (i + 1 < R && next_off(i) <= t0 + j) ++i;
        w[j] = expf(la[j] - lb[j]);
        k[j] = __ldg(coef + i) * w[j];
        local += static_cast<double>(k[j]);
      }
      *reinterpret_cast<float4*>(kappa + t0) = make_float4(k[0], k[1], k[2], k[3]);
      if (w_out != nullptr) *reinterpret_cast<float4*>(w_out + t0) = make_float4(w[0], w[1], w[2], w[3]);
    } else {
      for (int j = 0; j < 4 && t0 + j < n; ++j) {
        const int64_t t = t0 + j;
        while (i + 1 < R && next_off(i) <= t) ++i;
        const float w = expf(lp[t] - lp_roll[t]);
        const float k = __ldg(coef + i) * w;
        kappa[t] = k;
        if (w_out != nullptr) w_out[t] = w;
        local += static_cast<double>(k);
      }
    }
  }
  // fixed-order block reduction: warp butterfly, then warp partials in warp order
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = local;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < kKappaThreads / 32; ++w) s += warp_sums[w];
    block_sums[blockIdx.x] = s;
  }
}

// loss = sum of the block partials (fixed strided order, then a fixed tree).
__global__ void loss_final_kernel(const double* __restrict__ block_sums, int nb, float* __restrict__ loss) {
  __shared__ double sh[1024];
  double s = 0.0;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) s += block_sums[b];
  sh[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x >> 1; w > 0; w >>= 1) {
    if (threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = static_cast<float>(sh[0]);
}

// ------------------------------------------------------------------------ backward

// dZ[t, v] = kappa_t ([v == y_t] - 2^{(z - lse_t) log2 e}) for one chunk of rows,
// written as bf16 rows of stride ldz (columns >= V of the stride padding get 0).
struct EpiDz {
  const int32_t* ids;  // chunk-relative pointers
  const float* lse;
  const float* kappa;
  int64_t rows;        // valid rows in the chunk
  int V;
  int64_t ldz;         // row stride of dz in elements (V rounded up to 8)
  __nv_bfloat16* dz;

  struct State {
    float lse, kappa;
    int y;
    int64_t row;
  };

  __device__ __forceinline__ void begin_unit(State& st, int mb, int, int r) const {
    st.row = static_cast<int64_t>(mb) * BM + r;
    if (st.row < rows) {
      st.y = __ldg(ids + st.row);
      st.lse = __ldg(lse + st.row);
      st.kappa = __ldg(kappa + st.row);
    } else {
      st.y = -1;
      st.lse = 0.0f;
      st.kappa = 0.0f;
    }
  }

  __device__ __forceinline__ void tile(State& st, uint32_t taddr, int, int nt, int) const {
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int col0 = nt * BN + c * 32;
      if (col0 >= V) break;
      float v[32];
      __syncwarp();  // the TMEM load is warp-collective: reconverge first
      tmem_ld_32cols(taddr + c * 32, v);
      if (st.row < rows) {
      uint32_t packed[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        float g0 = st.kappa * ((col0 + j == st.y ? 1.0f : 0.0f) - ex2_approx((v[j] - st.lse) * kLog2e));
        float g1 = st.kappa * ((col0 + j + 1 == st.y ? 1.0f : 0.0f) - ex2_approx((v[j + 1] - st.lse) * kLog2e));
        if (col0 + j >= V) g0 = 0.0f;
        if (col0 + j + 1 >= V) g1 = 0.0f;
        packed[j >> 1] = pack_bf16x2(g0, g1);
      }
      uint4* dst = reinterpret_cast<uint4*>(dz + st.row * ldz + col0);
      const int64_t room = ldz - col0;  // multiple of 8 elements
      const int nvec = room >= 32 ? 4 : static_cast<int>(room >> 3);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < nvec) dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
      }
    }
  }

  __device__ __forceinline__ void end_unit(const State&, int, int, int) const {}
};

// Store a 128 x 256 fp32 accumulator tile as bf16 rows (dH).
struct EpiStoreBf16 {
  __nv_bfloat16* out;  // chunk-relative
  int64_t ld;
  int64_t rows;
  int ncols;

  struct State {
    int64_t row;
  };

  __device__ __forceinline__ void begin_unit(State& st, int mb, int, int r) const {
    st.row = static_cast<int64_t>(mb) * BM + r;
  }

  __device__ __forceinline__ void tile(State& st, uint32_t taddr, int, int nt, int) const {
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int col0 = nt * BN + c * 32;
      if (col0 >= ncols) break;
      float v[32];
      __syncwarp();  // the TMEM load is warp-collective: reconverge first
      tmem_ld_32cols(taddr + c * 32, v);
      if (st.row < rows) {
        uint4* dst = reinterpret_cast<uint4*>(out + st.row * ld + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                              pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
      }
    }
  }

  __device__ __forceinline__ void end_unit(const State&, int, int, int) const {}
};

// dW tile: out = (accumulate ? out : 0) + acc, fp32 (chunk contributions added in chunk order).
struct EpiAccF32 {
  float* out;
  int64_t ld;
  int64_t rows;
  int ncols;
  int accumulate;

  struct State {
    int64_t row;
  };

  __device__ __forceinline__ void begin_unit(State& st, int mb, int, int r) const {
    st.row = static_cast<int64_t>(mb) * BM + r;
  }

  __device__ __forceinline__ void tile(State& st, uint32_t taddr, int, int nt, int) const {
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int col0 = nt * BN + c * 32;
      if (col0 >= ncols) break;
      float v[32];
      __syncwarp();  // the TMEM load is warp-collective: reconverge first
      tmem_ld_32cols(taddr + c * 32, v);
      if (st.row >= rows) {
        // padding row of the last vocabulary block: nothing to store
      } else if (accumulate) {
        float4* dst = reinterpret_cast<float4*>(out + st.row * ld + col0);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 o = dst[q];
          dst[q] = make_float4(o.x + v[4 * q], o.y + v[4 * q + 1], o.z + v[4 * q + 2], o.w + v[4 * q + 3]);
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(out + st.row * ld + col0);
#pragma unroll
        for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      }
    }
  }

  __device__ __forceinline__ void end_unit(const State&, int, int, int) const {}
};

}  // namespace rz
