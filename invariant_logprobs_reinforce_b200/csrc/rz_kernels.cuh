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
#include <cuda_fp16.h>

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

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 p = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// ------------------------------------------------------------------------ forward

// Forward epilogue.  Per row and per 256-column tile: the tile maximum, then
// e_v = 2^((z_v - tile_max) log2 e) and their sum, folded into the row's running
// (max, sum) pair of the current vocabulary segment:
//   m' = max(m, tile_max);  s' = s 2^((m - m') log2 e) + tile_sum 2^((tile_max - m') log2 e)
// The sampled token's logit is picked out of the tile that holds it.  With STORE_P the
// e_v are also written (fp16, TMA store) together with the tile maximum, so the backward
// can form softmax probabilities without recomputing the logits; the log-sum-exp
// arithmetic is the same code either way, so both variants give the same lse bits.
template <bool STORE_P>
struct EpiLse {
  CUtensorMap p_map;  // STORE_P: fp16 [rows, V] (box 32 x 32, 64-byte swizzle)
  const int32_t* ids; // launch-relative
  int64_t rows;       // rows in this launch
  int V;
  int n_tiles;        // 256-column tiles over V
  float* part_m;      // [S][part_ld] running max of the segment
  float* part_s;      // [S][part_ld] sum of exp(z - max) over the segment
  int64_t part_ld;
  float* zy;          // [rows] logit of the sampled token
  float* tile_max;    // STORE_P: [rows][n_tiles]

  struct State {
    float m, s;
    int y;
    int64_t row;
  };

  __device__ __forceinline__ void begin_unit(State& st, int mb, int, int r) const {
    st.row = static_cast<int64_t>(mb) * BM + r;
    st.y = st.row < rows ? __ldg(ids + st.row) : -1;
    st.m = -INFINITY;
    st.s = 0.0f;
  }

  __device__ __forceinline__ void tile(State& st, uint32_t taddr, int mb, int nt, int r, int lane,
                                       WarpStage& stage) const {
    // pass 1: tile maximum over the valid columns
    float tmax = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int col0 = nt * BN + c * 32;
      if (col0 >= V) break;  // uniform across the warp
      float v[32];
      __syncwarp();  // the TMEM load is warp-collective: reconverge first
      tmem_ld_32cols(taddr + c * 32, v);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < V) tmax = fmaxf(tmax, v[j]);
    }
    // pass 2: exponentials relative to the tile maximum, their sum, the gather
    float tsum = 0.0f;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int col0 = nt * BN + c * 32;
      if (col0 >= V) break;
      float v[32];
      __syncwarp();
      tmem_ld_32cols(taddr + c * 32, v);
      const unsigned off = static_cast<unsigned>(st.y - col0);
      if (off < 32u) {
        float z = v[0];
#pragma unroll
        for (int j = 1; j < 32; ++j) z = (static_cast<unsigned>(j) == off) ? v[j] : z;
        zy[st.row] = z;
      }
      float e[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        e[j] = (col0 + j < V) ? ex2_approx((v[j] - tmax) * kLog2e) : 0.0f;
        tsum += e[j];
      }
      if constexpr (STORE_P) {
        uint4 row[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          row[q] = make_uint4(pack_half2(e[8 * q], e[8 * q + 1]), pack_half2(e[8 * q + 2], e[8 * q + 3]),
                              pack_half2(e[8 * q + 4], e[8 * q + 5]), pack_half2(e[8 * q + 6], e[8 * q + 7]));
        stage.store_rows(&p_map, lane, row, col0, mb * BM + (r - lane), rows);
      }
    }
    const float m_new = fmaxf(st.m, tmax);
    st.s = st.s * ex2_approx((st.m - m_new) * kLog2e) + tsum * ex2_approx((tmax - m_new) * kLog2e);
    st.m = m_new;
    if constexpr (STORE_P) {
      if (st.row < rows) tile_max[st.row * n_tiles + nt] = tmax;
    }
  }

  __device__ __forceinline__ void end_unit(const State& st, int, int nu, int) const {
    if (st.row < rows) {
      part_m[static_cast<int64_t>(nu) * part_ld + st.row] = st.m;
      part_s[static_cast<int64_t>(nu) * part_ld + st.row] = st.s;
    }
  }
};

// lse = M + log(sum_s s_s 2^{(m_s - M) log2 e}), segments merged in order s = 0..S-1.
// Pointers are launch-relative; the partials have row stride part_ld.
__global__ void merge_lse_kernel(const float* __restrict__ part_m, const float* __restrict__ part_s,
                                 int64_t part_ld, const float* __restrict__ zy, const int32_t* __restrict__ ids,
                                 int64_t n, int V, int S, float* __restrict__ lp, float* __restrict__ lse_out,
                                 int* status) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n) return;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, part_m[static_cast<int64_t>(s) * part_ld + t]);
  float sum = 0.0f;
  for (int s = 0; s < S; ++s)
    sum += part_s[static_cast<int64_t>(s) * part_ld + t] *
           ex2_approx((part_m[static_cast<int64_t>(s) * part_ld + t] - M) * kLog2e);
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

// First response of every 4096-token block of the loss stage (one thread per block).
__global__ void block_first_kernel(const int64_t* __restrict__ off, int R, int64_t n, int nblocks,
                                   int* __restrict__ first) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  first[b] = find_response(off, R, min(n - 1, static_cast<int64_t>(b) * kKappaBlockTokens));
}

// kappa_t = coef_i * exp(lp_t - lp_rollout_t) (ratio unclipped) for the 4096 tokens of
// block `block0 + blockIdx.x`; per-block partial sums of kappa in fp64 with a fixed
// reduction order.  The segment offsets from the block's first response on are staged
// in shared memory; every thread issues all of its loads before using any of them.
__global__ void __launch_bounds__(kKappaThreads)
    token_kappa_kernel(const float* __restrict__ lp, const float* __restrict__ lp_roll,
                       const int64_t* __restrict__ off, int R, const float* __restrict__ coef,
                       const int* __restrict__ block_first, int64_t n, int block0, int vec_ok,
                       float* __restrict__ kappa, float* __restrict__ w_out, double* __restrict__ block_sums) {
  __shared__ int64_t s_off[kKappaStagedOffsets + 1];
  __shared__ double warp_sums[kKappaThreads / 32];
  const int blk = block0 + blockIdx.x;
  const int64_t b0 = static_cast<int64_t>(blk) * kKappaBlockTokens;
  const int64_t b1 = min(n, b0 + kKappaBlockTokens);
  const int i0 = min(max(block_first[blk], 0), R - 1);
  const int cnt = min(kKappaStagedOffsets, R - i0);  // responses i0 .. i0+cnt-1 staged, plus the end of the last
  for (int k = threadIdx.x; k <= cnt; k += kKappaThreads) s_off[k] = off[i0 + k];

  const bool full = vec_ok && b1 - b0 == kKappaBlockTokens;
  float4 la[kKappaIters], lb[kKappaIters];
  if (full) {
#pragma unroll
    for (int it = 0; it < kKappaIters; ++it) {
      const int64_t t0 = b0 + it * (kKappaThreads * 4) + threadIdx.x * 4;
      la[it] = __ldg(reinterpret_cast<const float4*>(lp + t0));
      lb[it] = __ldg(reinterpret_cast<const float4*>(lp_roll + t0));
    }
  }
  __syncthreads();

  // offset of response i+1 (shared memory inside the staged range)
  auto next_off = [&](int i) -> int64_t {
    const int k = i + 1 - i0;
    return (k >= 0 && k <= cnt) ? s_off[k] : __ldg(off + i + 1);
  };
  // response owning token t
  auto locate = [&](int64_t t) -> int {
    if (t < s_off[0] || t >= s_off[cnt]) return find_response(off, R, t);
    int lo = 0, hi = cnt - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return i0 + lo;
  };

  double local = 0.0;
  if (full) {
#pragma unroll
    for (int it = 0; it < kKappaIters; ++it) {
      const int64_t t0 = b0 + it * (kKappaThreads * 4) + threadIdx.x * 4;
      int i = locate(t0);
      const float a4[4] = {la[it].x, la[it].y, la[it].z, la[it].w};
      const float b4[4] = {lb[it].x, lb[it].y, lb[it].z, lb[it].w};
      float w[4], k[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        while (i + 1 < R && next_off(i) <= t0 + j) ++i;
        w[j] = expf(a4[j] - b4[j]);
        k[j] = __ldg(coef + i) * w[j];
        local += static_cast<double>(k[j]);
      }
      __stcs(reinterpret_cast<float4*>(kappa + t0), make_float4(k[0], k[1], k[2], k[3]));
      if (w_out != nullptr) __stcs(reinterpret_cast<float4*>(w_out + t0), make_float4(w[0], w[1], w[2], w[3]));
    }
  } else {
    for (int it = 0; it < kKappaIters; ++it) {
      const int64_t t0 = b0 + it * (kKappaThreads * 4) + threadIdx.x * 4;
      if (t0 >= b1) break;
      int i = locate(t0);
      for (int j = 0; j < 4 && t0 + j < b1; ++j) {
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
    double sum = 0.0;
    for (int w = 0; w < kKappaThreads / 32; ++w) sum += warp_sums[w];
    block_sums[blk] = sum;
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

// dZ[t, v] = kappa_t ([v == y_t] - p_tv) in bf16, in place over the stored fp16
// e_tv = exp(z_tv - tile_max_t,tile) of the forward: p_tv = e_tv exp(tile_max - lse_t).
// At the sampled token the value is kappa_t (1 - exp(lp_t)) = -kappa_t expm1(lp_t), from
// the forward's fp32 logprob, so confident tokens keep their small (1 - p) exactly.
// Columns from V up to the row stride are written as 0.  One thread: 8 columns.
constexpr int kDzThreads = 256;
constexpr int kDzColsPerBlock = kDzThreads * 8;

__global__ void __launch_bounds__(kDzThreads)
    dz_from_p_kernel(const float* __restrict__ lse, const float* __restrict__ lp, const float* __restrict__ kappa,
                     const int32_t* __restrict__ ids, const float* __restrict__ tile_max, int n_tiles, int V,
                     int64_t ldz, uint16_t* __restrict__ buf) {
  const int64_t row = blockIdx.y;
  const int64_t col = static_cast<int64_t>(blockIdx.x) * kDzColsPerBlock + threadIdx.x * 8;
  if (col >= ldz) return;
  uint4* p = reinterpret_cast<uint4*>(buf + row * ldz + col);
  if (col >= V) {
    *p = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4 raw = *p;
  const float k = __ldg(kappa + row);
  const int y = __ldg(ids + row);
  const float scale = ex2_approx((__ldg(tile_max + row * n_tiles + col / BN) - __ldg(lse + row)) * kLog2e);
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t out[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 e = __half22float2(*reinterpret_cast<const __half2*>(&w[q]));
    const int64_t c0 = col + 2 * q;
    float g0 = -k * (e.x * scale);
    float g1 = -k * (e.y * scale);
    if (c0 == y) g0 = -k * expm1f(__ldg(lp + row));
    if (c0 + 1 == y) g1 = -k * expm1f(__ldg(lp + row));
    if (c0 >= V) g0 = 0.0f;
    if (c0 + 1 >= V) g1 = 0.0f;
    out[q] = pack_bf16x2(g0, g1);
  }
  *p = make_uint4(out[0], out[1], out[2], out[3]);
}

// dH tile: fp32 accumulator -> bf16, TMA-stored into a [rows, d] map of the chunk.
struct EpiDh {
  CUtensorMap out_map;  // bf16 [rows, d], box 32 x 32, 64-byte swizzle

  struct State {};

  __device__ __forceinline__ void begin_unit(State&, int, int, int) const {}

  __device__ __forceinline__ void tile(State&, uint32_t taddr, int mb, int nt, int r, int lane,
                                       WarpStage& stage) const {
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int col0 = nt * BN + c * 32;
      if (col0 >= out_cols) break;
      float v[32];
      __syncwarp();
      tmem_ld_32cols(taddr + c * 32, v);
      uint4 row[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        row[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                            pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
      stage.store_rows(&out_map, lane, row, col0, mb * BM + (r - lane), out_rows);
    }
  }

  __device__ __forceinline__ void end_unit(const State&, int, int, int) const {}

  int out_cols;
  int64_t out_rows;
};

// dW tile: fp32 accumulator TMA-stored (first chunk) or TMA-reduce-added (later chunks,
// in chunk order) into the [V, d] fp32 map; every element gets exactly one store or add
// per chunk, so the result is deterministic.
struct EpiDw {
  CUtensorMap out_map;  // fp32 [V, d], box 16 x 32, 64-byte swizzle
  int out_cols;
  int64_t out_rows;
  int accumulate;

  struct State {};

  __device__ __forceinline__ void begin_unit(State&, int, int, int) const {}

  __device__ __forceinline__ void tile(State&, uint32_t taddr, int mb, int nt, int r, int lane,
                                       WarpStage& stage) const {
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int col0 = nt * BN + c * 32;
      if (col0 >= out_cols) break;
      float v[32];
      __syncwarp();
      tmem_ld_32cols(taddr + c * 32, v);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint4 row[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          row[q] = make_uint4(__float_as_uint(v[16 * h + 4 * q]), __float_as_uint(v[16 * h + 4 * q + 1]),
                              __float_as_uint(v[16 * h + 4 * q + 2]), __float_as_uint(v[16 * h + 4 * q + 3]));
        stage.store_rows(&out_map, lane, row, col0 + 16 * h, mb * BM + (r - lane), out_rows, accumulate != 0);
      }
    }
  }

  __device__ __forceinline__ void end_unit(const State&, int, int, int) const {}
};

}  // namespace rz
