// rz_simt.cuh -- the SIMT kernels around the tensor-core contractions:
//
//   merge_lse_kernel        fixed-order merge of the per-segment (max, sum) pairs -> lse, lp
//   coef_*_kernel           group means, coef_i = -A_i / (N L_i)
//   block_first_kernel      first response of each 4096-token block
//   token_kappa_kernel      unclipped ratio and kappa per token, per-block loss partials
//   loss_final_kernel       fixed-order sum of the partials
//   dz_from_p_kernel        dZ = kappa (onehot - softmax) from the forward's exponentials
//
// Definitions follow "vLLM says aligned kernels make asynchronous RL stable at lag 64"
// (ainewsbites.com), section "REINFORCE Zero removes the mismatch first"; the fixed
// orders follow "vLLM Train-Inference Consistency Release Notes" (agentlenshq.com),
// section "Achieving Bitwise Consistency" (kernel determinism, batch independence).
#pragma once

#include "rz_epilogues.cuh"

namespace rz {

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

// Group means and the per-response coefficient coef_i = -A_i / (N L_i), in three short
// launches over responses and groups:
//   coef_runs_kernel   checks segments and group ids, flags group ids that are not
//                      non-decreasing, and lets the first response of each run of equal
//                      ids sum the run's rewards (the whole group when ids are sorted)
//   coef_groups_kernel only when ids are not sorted: each group scans all responses
//   coef_kernel        A_i = r_i - gsum/gcnt, coef_i
// Both ways add a group's rewards in response-index order (fp64), so both give the same
// bits.  flags[0] is the unsorted flag (cleared with the status word).
constexpr int kCoefThreads = 256;

__global__ void __launch_bounds__(kCoefThreads)
    coef_runs_kernel(const float* __restrict__ rewards, const int64_t* __restrict__ off,
                     const int32_t* __restrict__ gid, int R, int G, int64_t n, double* __restrict__ gsum,
                     int* __restrict__ gcnt, int* flags, int* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R) return;
  int bad = 0;
  if (i == 0 && (off[0] != 0 || off[R] != n)) bad |= kDevBadSegments;
  if (off[i + 1] <= off[i]) bad |= kDevBadSegments;
  const int g = gid[i];
  if (g < 0 || g >= G) bad |= kDevBadGroupId;
  if (bad) atomicOr(status, bad);
  if (i + 1 < R && gid[i + 1] < g) atomicOr(flags, 1);
  if ((i > 0 && gid[i - 1] == g) || g < 0 || g >= G) return;  // not the start of a valid run
  double sum = 0.0;
  int c = 0;
  for (int j = i; j < R && gid[j] == g; ++j) {
    sum += static_cast<double>(rewards[j]);
    ++c;
  }
  gsum[g] = sum;  // with sorted ids every group is one run, so one writer per group
  gcnt[g] = c;
}

__global__ void __launch_bounds__(kCoefThreads)
    coef_groups_kernel(const float* __restrict__ rewards, const int32_t* __restrict__ gid, int R, int G,
                       double* __restrict__ gsum, int* __restrict__ gcnt, const int* flags) {
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= G || *flags == 0) return;
  double sum = 0.0;
  int c = 0;
  for (int i = 0; i < R; ++i) {
    if (__ldg(gid + i) == g) {
      sum += static_cast<double>(__ldg(rewards + i));
      ++c;
    }
  }
  gsum[g] = sum;
  gcnt[g] = c;
}

__global__ void __launch_bounds__(kCoefThreads)
    coef_kernel(const float* __restrict__ rewards, const int64_t* __restrict__ off, const int32_t* __restrict__ gid,
                int R, int G, const double* __restrict__ gsum, const int* __restrict__ gcnt,
                float* __restrict__ coef) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R) return;
  const int g = gid[i];
  const int64_t L = off[i + 1] - off[i];
  if (g < 0 || g >= G || L <= 0 || gcnt[g] <= 0) {
    coef[i] = __int_as_float(0x7fc00000);
    return;
  }
  const double A = static_cast<double>(rewards[i]) - gsum[g] / static_cast<double>(gcnt[g]);
  coef[i] = static_cast<float>(-A / (static_cast<double>(R) * static_cast<double>(L)));
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

// kappa_t = coef_i * w_t with the unclipped ratio w_t = exp(lp_t - lp_rollout_t), for the
// 4096 tokens of block `block0 + blockIdx.x`; per-block partial sums of kappa with a fixed
// reduction order (each lane adds its 4 consecutive tokens in fp32, everything else in
// fp64).  Warp w owns the block's tokens [512 w, 512 w + 512) as four windows of 128
// (lane: 4 consecutive tokens, one 16-byte load per array).
//
// Fast path (every response touching the block staged: at most 256): the responses'
// starts relative to the block and their coefficients sit in shared memory; a lane
// finds its first token's response by a short walk and then advances with one compare
// per token (a boundary can only fall between two consecutive tokens).  Otherwise the
// block walks the global offsets.
__global__ void __launch_bounds__(kKappaThreads)
    token_kappa_kernel(const float* __restrict__ lp, const float* __restrict__ lp_roll,
                       const int64_t* __restrict__ off, int R, const float* __restrict__ coef,
                       const int* __restrict__ block_first, int64_t n, int block0, int vec_ok,
                       float* __restrict__ kappa, float* __restrict__ w_out, double* __restrict__ block_sums) {
  constexpr int kFar = 1 << 30;  // a relative start beyond the block
  __shared__ int s_rel[kKappaStagedOffsets + 1];  // start of staged response k, relative to the block
  __shared__ float s_coef[kKappaStagedOffsets];
  __shared__ double warp_sums[kKappaThreads / 32];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int blk = block0 + blockIdx.x;
  const int64_t b0 = static_cast<int64_t>(blk) * kKappaBlockTokens;
  const int nb = static_cast<int>(min(n - b0, static_cast<int64_t>(kKappaBlockTokens)));  // tokens in the block
  const int i0 = min(max(block_first[blk], 0), R - 1);
  const int cnt = min(kKappaStagedOffsets, R - i0);
  for (int k = threadIdx.x; k <= cnt; k += kKappaThreads) {
    const int64_t o = (i0 + k < R) ? off[i0 + k] - b0 : kFar;
    s_rel[k] = static_cast<int>(max(min(o, static_cast<int64_t>(kFar)), static_cast<int64_t>(-kFar)));
    if (k < cnt) s_coef[k] = coef[i0 + k];
  }
  const bool full = vec_ok && nb == kKappaBlockTokens;
  const int wrel = warp * (kKappaBlockTokens / 8);
  float4 la[kKappaIters], lb[kKappaIters];
  if (full) {
#pragma unroll
    for (int it = 0; it < kKappaIters; ++it) {
      const int64_t t0 = b0 + wrel + it * 128 + lane * 4;
      la[it] = __ldcs(reinterpret_cast<const float4*>(lp + t0));
      lb[it] = __ldcs(reinterpret_cast<const float4*>(lp_roll + t0));
    }
  }
  __syncthreads();
  // the staged responses cover the block when the first starts at or before its first
  // token and the one after the last staged starts at or after its end
  const bool staged = s_rel[0] <= 0 && s_rel[cnt] >= nb;

  double local = 0.0;
  if (staged && full) {
    int k = 0;  // staged response of the current token
#pragma unroll
    for (int it = 0; it < kKappaIters; ++it) {
      const int tr = wrel + it * 128 + lane * 4;
      while (s_rel[k + 1] <= tr) ++k;
      const float a4[4] = {la[it].x, la[it].y, la[it].z, la[it].w};
      const float b4[4] = {lb[it].x, lb[it].y, lb[it].z, lb[it].w};
      float w[4], kv[4];
      float part = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (j > 0 && s_rel[k + 1] <= tr + j) ++k;
        w[j] = ex2_approx((a4[j] - b4[j]) * kLog2e);
        kv[j] = s_coef[k] * w[j];
        part += kv[j];
      }
      const int64_t t0 = b0 + tr;
      __stcs(reinterpret_cast<float4*>(kappa + t0), make_float4(kv[0], kv[1], kv[2], kv[3]));
      if (w_out != nullptr) __stcs(reinterpret_cast<float4*>(w_out + t0), make_float4(w[0], w[1], w[2], w[3]));
      local += static_cast<double>(part);
    }
  } else {
    // general path: tail blocks, unaligned arrays, or more than 256 responses in the block
    for (int it = 0; it < kKappaIters; ++it) {
      const int64_t t0 = b0 + wrel + it * 128 + lane * 4;
      float part = 0.0f;
      if (t0 < b0 + nb) {
        int i = find_response(off, R, t0);
        for (int j = 0; j < 4 && t0 + j < b0 + nb; ++j) {
          const int64_t t = t0 + j;
          while (i + 1 < R && __ldg(off + i + 1) <= t) ++i;
          const float w = ex2_approx((lp[t] - lp_roll[t]) * kLog2e);
          const float kv = __ldg(coef + i) * w;
          kappa[t] = kv;
          if (w_out != nullptr) w_out[t] = w;
          part += kv;
        }
      }
      local += static_cast<double>(part);
    }
  }
  // fixed-order block reduction: warp butterfly, then warp partials in warp order
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if (lane == 0) warp_sums[warp] = local;
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
// Columns from V up to the row stride are written as 0.  One block per row; each thread
// converts 8 columns (16 bytes) at a time, four vectors in flight.
constexpr int kDzThreads = 256;
constexpr int kDzUnroll = 4;

__global__ void __launch_bounds__(kDzThreads)
    dz_from_p_kernel(const float* __restrict__ lse, const float* __restrict__ lp, const float* __restrict__ kappa,
                     const int32_t* __restrict__ ids, const float* __restrict__ tile_max, int n_tiles, int V,
                     int64_t ldz, uint16_t* __restrict__ buf) {
  const int64_t row = blockIdx.x;
  const float k = kappa[row];
  const int y = ids[row];
  const float l = lse[row];
  const float at_y = -k * expm1f(lp[row]);
  const float* tmax = tile_max + row * n_tiles;
  uint4* rowp = reinterpret_cast<uint4*>(buf + row * ldz);
  const int nvec = static_cast<int>(ldz / 8);
  const int vvalid = (V + 7) / 8;  // vectors holding at least one column < V
  constexpr int kStep = kDzThreads * kDzUnroll;
  for (int v0 = threadIdx.x; v0 < nvec; v0 += kStep) {
    uint4 raw[kDzUnroll];
#pragma unroll
    for (int u = 0; u < kDzUnroll; ++u) {
      const int v = v0 + u * kDzThreads;
      raw[u] = v < vvalid ? __ldcs(rowp + v) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kDzUnroll; ++u) {
      const int v = v0 + u * kDzThreads;
      if (v >= nvec) break;
      const int col = v * 8;
      uint4 out = make_uint4(0u, 0u, 0u, 0u);
      if (v < vvalid) {
        // dZ = -kappa * p = (-kappa * exp(tile_max - lse)) * e
        const float f = -k * ex2_approx((__ldg(tmax + col / BN) - l) * kLog2e);
        const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
        float g[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 e = __half22float2(*reinterpret_cast<const __half2*>(&w[q]));
          g[2 * q] = e.x * f;
          g[2 * q + 1] = e.y * f;
        }
        if (static_cast<unsigned>(y - col) < 8u) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (col + j == y) g[j] = at_y;
        }
        if (col + 8 > V) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (col + j >= V) g[j] = 0.0f;
        }
        out = make_uint4(pack_bf16x2(g[0], g[1]), pack_bf16x2(g[2], g[3]), pack_bf16x2(g[4], g[5]),
                         pack_bf16x2(g[6], g[7]));
      }
      __stcs(rowp + v, out);
    }
  }
}

}  // namespace rz
