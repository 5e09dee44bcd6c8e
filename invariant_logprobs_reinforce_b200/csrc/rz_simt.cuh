// rz_simt.cuh -- the SIMT kernels around the tensor-core contractions:
//
//   merge_lse_kernel        fixed-order merge of the per-segment (max, sum) pairs -> lse, lp
//   loss_setup_kernel       device checks, group means, coef_i = -A_i / (N L_i), the first
//                           response of each 4096-token block
//   token_kappa_kernel      unclipped ratio and kappa per token, per-block loss partials, and
//                           (its last block) their fixed-order sum, the loss
//   dz_from_p_kernel        dZ = kappa (onehot - softmax) from the forward's exponentials
//   masked_count_kernel, gate_kernel
//                           loss-stage options: counted tokens per response under a token
//                           mask; the sequence gate on the geometric-mean ratio
//   ratio_stats_*, response_mean_ratio_kernel
//                           ratio diagnostics: KL estimators, min / max / deviation peak and
//                           exact lower median (radix select), per-response mean ratio
//   sumsq_kernel, sqrt_sum_kernel
//                           gradient norms (fixed-order fp64 reductions)
//   quantize_rows_e4m3_kernel
//                           per-row e4m3 codes and scales for the fp8 forward
//   sum_shards_kernel       rank-order sum of stacked shards (deterministic all-reduce)
//   wait_timeout_selftest_kernel
//                           the bounded mbarrier wait on a barrier nothing arrives on
//
// Definitions follow "vLLM says aligned kernels make asynchronous RL stable at lag 64"
// (ainewsbites.com), section "REINFORCE Zero removes the mismatch first"; the fixed
// orders follow "vLLM Train-Inference Consistency Release Notes" (agentlenshq.com),
// section "Achieving Bitwise Consistency" (kernel determinism, batch independence).
#pragma once

#include <cuda_fp8.h>

#include "rz_epilogues.cuh"

namespace rz {

// lse = M + log(sum_s s_s 2^{(m_s - M) log2 e}), segments merged in order s = 0..S-1.
// Pointers are launch-relative; the partials have row stride part_ld.
//
// n_tiles > 0: the partials are per 256-column tile (calls with too few row blocks to fill
// the GPU with one unit per segment run one unit per tile) and each segment's pair is first
// rebuilt by folding its tiles' pairs in order with lse_fold, exactly as the epilogue folds
// them when a unit is a whole segment: the same bits either way.
//
// If a wait of an earlier kernel of the same call gave up (the timeout bit of the status
// word is set), some partials were never written and may hold an earlier call's values:
// every lp and lse of the launch is then NaN instead of a plausible wrong number.
__global__ void merge_lse_kernel(const float* __restrict__ part_m, const float* __restrict__ part_s,
                                 int64_t part_ld, const float* __restrict__ zy, const int32_t* __restrict__ ids,
                                 int64_t n, int V, int S, float* __restrict__ lp, float* __restrict__ lse_out,
                                 int* status, int n_tiles = 0) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n) return;
  if (*reinterpret_cast<volatile const int*>(status) & kDevWaitTimeout) {
    lp[t] = __int_as_float(0x7fc00000);
    if (lse_out != nullptr) lse_out[t] = __int_as_float(0x7fc00000);
    return;
  }
  // pair of segment s: stored, or folded from its tiles
  auto segment = [&](int s, float& m, float& sm) {
    if (n_tiles == 0) {
      m = part_m[static_cast<int64_t>(s) * part_ld + t];
      sm = part_s[static_cast<int64_t>(s) * part_ld + t];
      return;
    }
    m = -INFINITY;
    sm = 0.0f;
    for (int k = s * kSegTiles; k < min(n_tiles, (s + 1) * kSegTiles); ++k)
      lse_fold(m, sm, part_m[static_cast<int64_t>(k) * part_ld + t], part_s[static_cast<int64_t>(k) * part_ld + t]);
  };
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) {
    float m, sm;
    segment(s, m, sm);
    M = fmaxf(M, m);
  }
  float sum = 0.0f;
  for (int s = 0; s < S; ++s) {
    float m, sm;
    segment(s, m, sm);
    sum += sm * ex2_approx((m - M) * kLog2e);
  }
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

// Group means and the per-response coefficient coef_i = -A_i / (N L_i): loss_setup_kernel
// below.  flags[0] is the unsorted-ids flag; flags[1] and flags[2] are the tickets of the
// setup kernel and of the ratio / kappa kernel (all cleared with the status word).

// Per response (one warp each): the number of tokens whose mask byte is non-zero.  The
// 16-byte-aligned middle of the response's mask is read 16 bytes per lane (nonzero bytes
// counted four at a time: __vcmpne4 sets a byte to 0xff where it is nonzero), the ragged ends
// byte by byte; the count is an integer, so the split does not change it.
__device__ __forceinline__ int nonzero_bytes(uint32_t x) { return __popc(__vcmpne4(x, 0u)) >> 3; }

__global__ void __launch_bounds__(256)
    masked_count_kernel(const uint8_t* __restrict__ mask, const int64_t* __restrict__ off, int R,
                        int* __restrict__ counted) {
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= R) return;
  const int64_t o0 = off[i], o1 = off[i + 1];
  const uint64_t base = reinterpret_cast<uint64_t>(mask);
  const int64_t a0 = min(o1, o0 + static_cast<int64_t>((16u - ((base + static_cast<uint64_t>(o0)) & 15u)) & 15u));
  const int64_t a1 = a0 + ((o1 - a0) & ~int64_t{15});
  int c = 0;
  for (int64_t t = o0 + lane; t < a0; t += 32) c += mask[t] != 0;
  for (int64_t t = a0 + 16 * lane; t < a1; t += 16 * 32) {
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(mask + t));
    c += nonzero_bytes(v.x) + nonzero_bytes(v.y) + nonzero_bytes(v.z) + nonzero_bytes(v.w);
  }
  for (int64_t t = a1 + lane; t < o1; t += 32) c += mask[t] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) counted[i] = c;
}

// Sequence gate (one warp per response): the response's geometric-mean ratio
// exp(mean over its counted tokens of (lp - lp_rollout)); outside [lo, hi] the response's
// coefficient becomes 0.  Lane-strided fp64 partials and a fixed butterfly: deterministic.
__global__ void __launch_bounds__(256)
    gate_kernel(const float* __restrict__ lp, const float* __restrict__ lp_roll, const uint8_t* __restrict__ mask,
                const int64_t* __restrict__ off, int R, double lo, double hi, float* __restrict__ coef) {
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= R) return;
  double sum = 0.0;
  int c = 0;
  for (int64_t t = off[i] + lane; t < off[i + 1]; t += 32) {
    if (mask != nullptr && mask[t] == 0) continue;
    sum += static_cast<double>(lp[t]) - static_cast<double>(lp_roll[t]);
    ++c;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
  }
  if (lane == 0 && c > 0) {
    const double g = exp(sum / c);
    if (!(g >= lo && g <= hi)) coef[i] = 0.0f;
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

// The loss stage's setup in one launch:
//  - thread i < R checks response i (segments, group id) and flags ids that are not
//    non-decreasing;
//  - coef_i = -A_i / (N L_i) from the sum of the rewards of the run of equal valid ids that
//    holds response i, added in response order from the run's first response (with
//    non-decreasing ids a run is the whole group); the run's first response also writes the
//    group's sum and count.  A warp covers 32 consecutive responses and loads their fields
//    at once; a run inside the window is summed from registers (shuffles, in order), and
//    only a run that crosses the window's edge reads the neighbouring responses, 32 at a
//    time;
//  - thread i < R writes i as the first response of every 4096-token block that starts
//    inside response i (after a failed segment check some blocks may keep stale entries;
//    the ratio / kappa kernel clamps what it reads, and the outputs carry no meaning then);
//  - the last block to finish (a ticket on `ticket`, cleared with the status word) redoes
//    the group sums by scanning the responses in index order and rewrites every coef when
//    the ids were not sorted.  Either way a group's rewards are added in response order
//    from 0, so both give the same bits.
// counted (nullable): tokens per response under a token mask (masked_count_kernel).
constexpr int kSetupThreads = 256;

// coef_i from response i's reward, counted length L, validity and its group's (sum, count)
__device__ __forceinline__ float coef_of(float reward, int64_t L, bool bad, double gsum_g, int gcnt_g, double N) {
  if (bad || gcnt_g <= 0) return __int_as_float(0x7fc00000);
  if (L <= 0) return 0.0f;  // every token of the response is masked out: it contributes nothing
  const double A = static_cast<double>(reward) - gsum_g / static_cast<double>(gcnt_g);
  return static_cast<float>(-A / (N * static_cast<double>(L)));
}

__device__ __forceinline__ float response_coef(const float* __restrict__ rewards, const int64_t* __restrict__ off,
                                               const int32_t* __restrict__ gid, int G, double N,
                                               const int* __restrict__ counted, double gsum_g, int gcnt_g, int i) {
  const int g = gid[i];
  const int64_t L = counted != nullptr ? counted[i] : off[i + 1] - off[i];
  return coef_of(rewards[i], L, g < 0 || g >= G || off[i + 1] <= off[i], gsum_g, gcnt_g, N);
}

__global__ void __launch_bounds__(kSetupThreads)
    loss_setup_kernel(const float* __restrict__ rewards, const int64_t* __restrict__ off,
                      const int32_t* __restrict__ gid, int R, int G, int64_t n, double N,
                      const int* __restrict__ counted, double* __restrict__ gsum, int* __restrict__ gcnt,
                      float* __restrict__ coef, int nblocks, int* __restrict__ bfirst, int* flags, int* ticket,
                      int* status) {
  __shared__ bool s_last;
  // the kappa kernel that follows may start launching now: it waits for this grid to
  // finish before it reads anything written here
  grid_dependents_launch();
  constexpr unsigned kAll = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int w0 = i - lane;  // the warp's first response
  const bool in = i < R;
  // every field of response i, loaded at once
  const int g = in ? gid[i] : 0;
  const bool has_next = in && i + 1 < R;
  const int g_next = has_next ? gid[i + 1] : 0;
  const int g_prev = (lane == 0 && in && i > 0) ? gid[i - 1] : 0;
  const float r = in ? rewards[i] : 0.0f;
  const int64_t o0 = in ? off[i] : 0, o1 = in ? off[i + 1] : 0;
  const int64_t L = (in && counted != nullptr) ? counted[i] : o1 - o0;
  const bool gvalid = in && g >= 0 && g < G;
  if (in) {
    int bad = 0;
    if (i == 0 && (o0 != 0 || off[R] != n)) bad |= kDevBadSegments;
    if (o1 <= o0) bad |= kDevBadSegments;
    if (!gvalid) bad |= kDevBadGroupId;
    if (bad) atomicOr(status, bad);
    if (has_next && g_next < g) atomicOr(flags, 1);
  }
  // runs of equal valid ids in the window: a lane starts one when its id differs from the
  // previous response's (lane 0: from response w0 - 1); an invalid or absent response
  // breaks every run
  const int g_left = __shfl_up_sync(kAll, g, 1);
  const bool brk = !gvalid || (lane == 0 ? (i == 0 || g_prev != g) : g_left != g);
  const unsigned B = __ballot_sync(kAll, brk);
  const unsigned upto = B & (kAll >> (31 - lane));  // starts at lanes <= lane
  const unsigned above = B & ~(kAll >> (31 - lane));
  const int ls = upto ? 31 - __clz(upto) : 0;  // the lane's run, clipped to the window
  const int le = above ? __ffs(above) - 2 : 31;
  // the run of lane 0, if it began in an earlier window: its responses before w0, in order
  double sum = 0.0;
  int c = 0;
  if (__shfl_sync(kAll, gvalid && !brk, 0)) {
    const int g0 = __shfl_sync(kAll, g, 0);
    int start = w0;
    for (int base = w0 - 32;; base -= 32) {  // its first response, 32 at a time
      const int j = base + lane;
      const unsigned m = __ballot_sync(kAll, !(j >= 0 && gid[j] == g0));
      if (m) {
        start = base + 32 - __clz(m);
        break;
      }
    }
    double acc = 0.0;
    for (int base = start; base < w0; base += 32) {
      const int j = base + lane;
      const float rj = j < w0 ? rewards[j] : 0.0f;
      const int nk = min(32, w0 - base);
      for (int k = 0; k < 32; ++k) {
        const float v = __shfl_sync(kAll, rj, k);
        if (k < nk) acc += static_cast<double>(v);
      }
    }
    if (upto == 0) {  // the lanes of that run
      sum = acc;
      c = w0 - start;
    }
  }
  // the window's part of the lane's run, in order
  for (int k = 0; k < 32; ++k) {
    const float v = __shfl_sync(kAll, r, k);
    if (k >= ls && k <= le) sum += static_cast<double>(v);
  }
  c += le - ls + 1;
  // the run of lane 31, if it goes on past the window: its responses after, in order
  if (__shfl_sync(kAll, gvalid && has_next && g_next == g, 31)) {
    const int g31 = __shfl_sync(kAll, g, 31);
    const bool last_run = le == 31;
    for (int base = w0 + 32;; base += 32) {
      const int j = base + lane;
      const bool same = j < R && gid[j] == g31;
      const float rj = j < R ? rewards[j] : 0.0f;
      const unsigned m = __ballot_sync(kAll, !same);
      const int nk = m ? __ffs(m) - 1 : 32;
      for (int k = 0; k < 32; ++k) {
        const float v = __shfl_sync(kAll, rj, k);
        if (last_run && k < nk) sum += static_cast<double>(v);
      }
      if (last_run) c += nk;
      if (nk < 32) break;
    }
  }
  if (in) {
    if (gvalid && brk) {  // the run's first response; with sorted ids one writer per group
      gsum[g] = sum;
      gcnt[g] = c;
    }
    coef[i] = coef_of(r, L, !gvalid || o1 <= o0, sum, c, N);
  }
  // first responses of the 4096-token blocks: block b starts at token b * 4096, which lies in
  // the response i with off[i] <= b * 4096 < off[i + 1], i.e. b in [ceil(off[i] / 4096),
  // ceil(off[i + 1] / 4096)); with valid offsets every block is written once, by that response
  if (in) {
    const int64_t b_hi = min(static_cast<int64_t>(nblocks), (o1 + kKappaBlockTokens - 1) / kKappaBlockTokens);
    for (int64_t b = max(static_cast<int64_t>(0), (o0 + kKappaBlockTokens - 1) / kKappaBlockTokens); b < b_hi; ++b)
      bfirst[b] = i;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1) == static_cast<int>(gridDim.x) - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (*reinterpret_cast<volatile const int*>(flags) == 0) return;  // sorted: every coef is written
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    double sum = 0.0;
    int c = 0;
    for (int j = 0; j < R; ++j) {
      if (__ldg(gid + j) == g) {
        sum += static_cast<double>(__ldg(rewards + j));
        ++c;
      }
    }
    gsum[g] = sum;
    gcnt[g] = c;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < R; j += blockDim.x) {
    const int g = gid[j];
    const bool valid = g >= 0 && g < G;
    coef[j] = response_coef(rewards, off, gid, G, N, counted, valid ? gsum[g] : 0.0, valid ? gcnt[g] : 0, j);
  }
}

// kappa_t = coef_i * w_t with the unclipped ratio w_t = exp(lp_t - lp_rollout_t) over the
// 4096-token blocks [block0, block0 + nblk), per-block partial sums of kappa with a fixed
// reduction order (each lane adds its 4 consecutive tokens in fp32, everything else in
// fp64), and (the CTA that finishes last of all the call's blocks) their fixed-order sum,
// the loss.  Warp w owns a block's tokens [512 w, 512 w + 512) as four windows of 128 (lane:
// 4 consecutive tokens).
//
// Persistent CTAs, a few per SM, each taking the blocks blockIdx.x, blockIdx.x + gridDim.x,
// ...: thread 0 streams a whole block's lp, lp_rollout (and mask) into shared memory with
// bulk copies, KappaSmem::kStages blocks ahead, so the memory system always has several blocks in
// flight however long the arithmetic of one takes.  The responses touching a block (their
// starts relative to the block and their coefficients, at most 256 staged) are fetched one
// block ahead into registers and put into shared memory when the block begins (two buffers by
// block parity, so that one barrier per block suffices: after it, thread 0 adds the previous
// block's warp partials and refills the previous block's stage); a lane finds
// its first token's response by a short walk and then advances with one compare per token
// (a boundary can only fall between two consecutive tokens).  A block that is not whole or
// not 16-byte aligned, or that more than 256 responses touch, takes the general path from
// global memory.  A block's partial is computed the same way whichever CTA takes it, so the
// loss does not depend on the grid.
// MASKED / CLIPPED: compiled variants with and without the token mask and the truncated-IS
// cap, so the plain call carries neither per-token test (the arithmetic is the same).
constexpr int kKappaMaxStages = 3;

// Unmasked: three CTAs per SM with two stages each; masked (a ninth byte per token): two CTAs
// with three stages (three CTAs would not fit).  Six blocks in flight per SM either way.
template <bool MASKED>
struct KappaSmem {
  static constexpr int kStages = MASKED ? 3 : 2;
  static constexpr int kCtasPerSm = MASKED ? 2 : 3;
  static constexpr int kStageBytes = kKappaBlockTokens * (8 + (MASKED ? 1 : 0));  // lp | lp_rollout | mask
  static constexpr int kBytes = kStages * kStageBytes + 8 * kStages;              // + one barrier per stage
};
static_assert(KappaSmem<true>::kStageBytes % 16 == 0 && 4 * kKappaBlockTokens % 16 == 0, "bulk copy sizes");

// Staged responses of one block, fetched into registers ahead of their use: thread t holds
// entry t (start and coefficient of response i0 + t), thread 0 also entry 256's start.
struct KappaStaging {
  int i0, cnt;
  int64_t o, o_last;
  float c;
};

__device__ __forceinline__ void kappa_staging_fetch(const int64_t* __restrict__ off, const float* __restrict__ coef,
                                                    int R, int first, KappaStaging& st) {
  constexpr int64_t kFarAbs = int64_t{1} << 62;  // a start beyond every block
  const int t = threadIdx.x;
  st.i0 = min(max(first, 0), R - 1);
  st.cnt = min(kKappaStagedOffsets, R - st.i0);
  st.o = (t <= st.cnt && st.i0 + t < R) ? off[st.i0 + t] : kFarAbs;
  st.c = t < st.cnt ? coef[st.i0 + t] : 0.0f;
  st.o_last = (t == 0 && st.cnt == kKappaStagedOffsets && st.i0 + kKappaStagedOffsets < R)
                  ? off[st.i0 + kKappaStagedOffsets]
                  : kFarAbs;
}

template <bool MASKED, bool CLIPPED>
__global__ void __launch_bounds__(kKappaThreads, KappaSmem<MASKED>::kCtasPerSm)
    token_kappa_kernel(const float* __restrict__ lp, const float* __restrict__ lp_roll,
                       const int64_t* __restrict__ off, int R, const float* __restrict__ coef,
                       const int* __restrict__ block_first, int64_t n, int block0, int nblk, int vec_ok,
                       const uint8_t* __restrict__ mask, float clip_max, float* __restrict__ kappa,
                       float* __restrict__ w_out, double* __restrict__ block_sums, int total_blocks,
                       int* __restrict__ ticket, float* __restrict__ loss, int* status) {
  using Smem = KappaSmem<MASKED>;
  constexpr int kS = Smem::kStages;
  constexpr int kFar = 1 << 30;  // a relative start beyond the block
  extern __shared__ __align__(128) uint8_t kx_smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(kx_smem + kS * Smem::kStageBytes);
  // double-buffered by block parity, so that one barrier per block suffices
  __shared__ int s_rel[2][kKappaStagedOffsets + 1];  // start of staged response k, relative to the block
  __shared__ float s_coef[2][kKappaStagedOffsets];
  __shared__ double warp_sums[2][kKappaThreads / 32];
  __shared__ bool s_last;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int wrel = warp * (kKappaBlockTokens / (kKappaThreads / 32));
  const int my_blocks =
      static_cast<int>(blockIdx.x) < nblk ? (nblk - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x : 0;
  auto blk_of = [&](int k) { return block0 + static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x); };
  auto streamed = [&](int blk) {
    return vec_ok != 0 && static_cast<int64_t>(blk + 1) * kKappaBlockTokens <= n;
  };
  auto stage_ptr = [&](int k) { return kx_smem + (k % kS) * Smem::kStageBytes; };
  const uint64_t pol = make_l2_policy<kL2EvictFirst>();
  auto issue = [&](int k) {  // thread 0: bulk copies of this CTA's k-th block into its stage
    const int blk = blk_of(k);
    if (!streamed(blk)) return;
    uint8_t* sp = stage_ptr(k);
    uint64_t* bar = &full[k % kS];
    const int64_t b0 = static_cast<int64_t>(blk) * kKappaBlockTokens;
    mbar_arrive_expect_tx(bar, Smem::kStageBytes);
    bulk_load_1d(sp, lp + b0, 4 * kKappaBlockTokens, bar, pol);
    bulk_load_1d(sp + 4 * kKappaBlockTokens, lp_roll + b0, 4 * kKappaBlockTokens, bar, pol);
    if constexpr (MASKED) bulk_load_1d(sp + 8 * kKappaBlockTokens, mask + b0, kKappaBlockTokens, bar, pol);
  };
  if (tid == 0) {
    for (int s = 0; s < kS; ++s) mbar_init(&full[s], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (tid == 0)
    for (int k = 0; k < min(kS, my_blocks); ++k) issue(k);
  // launched as a programmatic dependent of the setup kernel, the copies above overlap the
  // setup; everything below reads what the setup wrote
  grid_dependency_wait();

  KappaStaging cur{};
  int first_next = 0;
  if (my_blocks > 0) kappa_staging_fetch(off, coef, R, block_first[blk_of(0)], cur);
  if (my_blocks > 1) first_next = block_first[blk_of(1)];
  bool aborted = false;
  int k = 0;
  for (; k < my_blocks; ++k) {
    const int blk = blk_of(k);
    const int64_t b0 = static_cast<int64_t>(blk) * kKappaBlockTokens;
    const int nb = static_cast<int>(min(n - b0, static_cast<int64_t>(kKappaBlockTokens)));  // tokens in the block
    // this block's responses into the staging buffer of its parity (its last readers, block
    // k - 2, are past the barrier of block k - 1)
    const int pb = k & 1;
    if (tid <= cur.cnt)
      s_rel[pb][tid] = static_cast<int>(max(min(cur.o - b0, static_cast<int64_t>(kFar)), static_cast<int64_t>(-kFar)));
    if (tid < cur.cnt) s_coef[pb][tid] = cur.c;
    if (tid == 0 && cur.cnt == kKappaStagedOffsets)
      s_rel[pb][kKappaStagedOffsets] =
          static_cast<int>(max(min(cur.o_last - b0, static_cast<int64_t>(kFar)), static_cast<int64_t>(-kFar)));
    // the next block's responses, and the one after's first response, fetched now
    KappaStaging nxt{};
    int first_after = 0;
    if (k + 1 < my_blocks) kappa_staging_fetch(off, coef, R, first_next, nxt);
    if (k + 2 < my_blocks) first_after = block_first[blk_of(k + 2)];
    const bool in_smem = streamed(blk);
    bool ok = true;
    if (in_smem) ok = mbar_wait(&full[k % kS], static_cast<uint32_t>((k / kS) & 1), nullptr);
    // the one barrier of a block: its staging is visible, and every thread is done with block
    // k - 1 (its stage may be refilled, its warp partials added)
    if (!__syncthreads_and(ok)) {  // a copy that never landed: give up on the launch
      aborted = true;
      break;
    }
    if (tid == 0 && k > 0) {
      double sum = 0.0;
      for (int w = 0; w < kKappaThreads / 32; ++w) sum += warp_sums[pb ^ 1][w];
      block_sums[blk_of(k - 1)] = sum;
      if (k - 1 + kS < my_blocks) issue(k - 1 + kS);
    }
    const int* rel = s_rel[pb];
    const float* cf = s_coef[pb];
    const int cnt = cur.cnt;
    // the staged responses cover the block when the first starts at or before its first
    // token and the one after the last staged starts at or after its end
    const bool staged = rel[0] <= 0 && rel[cnt] >= nb;
    double local = 0.0;
    if (staged && in_smem) {
      const uint8_t* sp = stage_ptr(k);
      const float* s_lp = reinterpret_cast<const float*>(sp);
      const float* s_lr = reinterpret_cast<const float*>(sp + 4 * kKappaBlockTokens);
      // staged response kr of the current token, the start of response kr + 1 and its coef
      // in registers: a token that starts no new response reads no shared memory for it
      int kr = 0;
      int next = rel[1];
      float ck = cf[0];
#pragma unroll
      for (int it = 0; it < kKappaIters; ++it) {
        const int tr = wrel + it * 128 + lane * 4;
        if (next <= tr) {
          do ++kr; while (rel[kr + 1] <= tr);
          next = rel[kr + 1];
          ck = cf[kr];
        }
        const float4 la = *reinterpret_cast<const float4*>(s_lp + tr);
        const float4 lb = *reinterpret_cast<const float4*>(s_lr + tr);
        const uint32_t m4 = MASKED ? *reinterpret_cast<const uint32_t*>(sp + 8 * kKappaBlockTokens + tr) : 0x01010101u;
        const float a4[4] = {la.x, la.y, la.z, la.w};
        const float b4[4] = {lb.x, lb.y, lb.z, lb.w};
        float w[4], kv[4];
        float part = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (j > 0 && next <= tr + j) {  // responses are non-empty: at most one start per token
            ++kr;
            next = rel[kr + 1];
            ck = cf[kr];
          }
          w[j] = ex2_approx((a4[j] - b4[j]) * kLog2e);
          const float g = CLIPPED ? fminf(w[j], clip_max) : w[j];
          kv[j] = (!MASKED || ((m4 >> (8 * j)) & 0xffu)) ? ck * g : 0.0f;
          part += kv[j];
        }
        const int64_t t0 = b0 + tr;
        __stcs(reinterpret_cast<float4*>(kappa + t0), make_float4(kv[0], kv[1], kv[2], kv[3]));
        if (w_out != nullptr) __stcs(reinterpret_cast<float4*>(w_out + t0), make_float4(w[0], w[1], w[2], w[3]));
        local += static_cast<double>(part);
      }
    } else {
      // general path: a partial or unaligned block, or more than 256 responses in the block
      for (int it = 0; it < kKappaIters; ++it) {
        const int64_t t0 = b0 + wrel + it * 128 + lane * 4;
        float part = 0.0f;
        if (t0 < b0 + nb) {
          int i = find_response(off, R, t0);
          for (int j = 0; j < 4 && t0 + j < b0 + nb; ++j) {
            const int64_t t = t0 + j;
            while (i + 1 < R && __ldg(off + i + 1) <= t) ++i;
            const float w = ex2_approx((lp[t] - lp_roll[t]) * kLog2e);
            const float g = CLIPPED ? fminf(w, clip_max) : w;
            const float kv = (!MASKED || mask[t] != 0) ? __ldg(coef + i) * g : 0.0f;
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
    if (lane == 0) warp_sums[pb][warp] = local;  // added in warp order after the next barrier
    cur = nxt;
    first_next = first_after;
  }
  __syncthreads();
  if (!aborted && tid == 0 && my_blocks > 0) {  // the last block's partial
    double sum = 0.0;
    for (int w = 0; w < kKappaThreads / 32; ++w) sum += warp_sums[(my_blocks - 1) & 1][w];
    block_sums[blk_of(my_blocks - 1)] = sum;
  }
  if (aborted && tid == 0) {
    atomicOr(status, kDevWaitTimeout);
    // copies still in flight must land before the CTA's shared memory goes away: block j < k
    // + kS - 1 was issued by the time the barrier of block k gave up
    const int issued_end = min(k == 0 ? kS : k - 1 + kS, my_blocks);
    for (int j = k; j < issued_end; ++j)
      if (streamed(blk_of(j))) mbar_wait(&full[j % kS], static_cast<uint32_t>((j / kS) & 1), nullptr);
  }
  // the CTA whose blocks complete the count over every launch of the call (the ticket is
  // cleared with the status word) forms the loss; a CTA that gave up still counts its
  // blocks, and the loss is then NaN
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(ticket, my_blocks) + my_blocks == total_blocks;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (*reinterpret_cast<volatile const int*>(status) & kDevWaitTimeout) {
    if (tid == 0) *loss = __int_as_float(0x7fc00000);
    return;
  }
  // loss = sum of the block partials in a fixed order: strided per thread, then a fixed tree
  // (in the stage memory, whose copies have all landed)
  double* s_tree = reinterpret_cast<double*>(kx_smem);
  double acc = 0.0;
  for (int b = tid; b < total_blocks; b += kKappaThreads) acc += __ldcg(block_sums + b);
  s_tree[tid] = acc;
  __syncthreads();
  for (int w = kKappaThreads >> 1; w > 0; w >>= 1) {
    if (tid < w) s_tree[tid] += s_tree[tid + w];
    __syncthreads();
  }
  if (tid == 0) *loss = static_cast<float>(s_tree[0]);
}

// ------------------------------------------------------------------------ backward

// ------------------------------------------------------------------------ fp8 operands
//
// Per-row e4m3 quantisation of a bf16 matrix (one block per row): scale = max|x| / 448
// (1 for an all-zero row), q = e4m3(x / scale) rounded to nearest even with saturation.
// x / scale and max|x| / 448 are IEEE fp32 divisions, so the codes are reproducible bit
// for bit by any fp32 implementation of the same two steps.
constexpr float kE4m3Max = 448.0f;

__global__ void __launch_bounds__(256)
    quantize_rows_e4m3_kernel(const __nv_bfloat16* __restrict__ X, int d, uint8_t* __restrict__ Q,
                              float* __restrict__ scale) {
  __shared__ float s_max[8];
  const int64_t row = blockIdx.x;
  const __nv_bfloat16* x = X + row * d;
  float m = 0.0f;
  for (int k = threadIdx.x; k < d; k += blockDim.x) m = fmaxf(m, fabsf(__bfloat162float(x[k])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = m;
  __syncthreads();
  m = s_max[0];
  for (int w = 1; w < 8; ++w) m = fmaxf(m, s_max[w]);
  const float sc = m > 0.0f ? __fdiv_rn(m, kE4m3Max) : 1.0f;
  if (threadIdx.x == 0) scale[row] = sc;
  for (int k = threadIdx.x; k < d; k += blockDim.x)
    Q[row * d + k] = __nv_cvt_float_to_fp8(__fdiv_rn(__bfloat162float(x[k]), sc), __NV_SATFINITE, __NV_E4M3);
}

// ------------------------------------------------------------------------ self-test
//
// The bounded-wait path of every kernel here, exercised on its own: one thread waits on an
// mbarrier that nothing arrives on, with the given limit; the wait gives up, the kernel
// sets the timeout status bit and records how long it waited, and returns normally.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns, int* status, unsigned long long* waited_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbarrier_init();
  const uint64_t t0 = global_timer_ns();
  const bool ok = mbar_wait(&bar, 0, nullptr, limit_ns);  // phase 0 never completes
  *waited_ns = global_timer_ns() - t0;
  if (!ok) atomicOr(status, kDevWaitTimeout);
}

// ------------------------------------------------------------------------ cross-GPU sum
//
// out[i] = sum over r = 0 .. nshards-1, in that order, of stacked[r * count + i]
// (fp64 accumulation, one rounding to fp32): the reduction step of a data-parallel
// all-reduce whose result does not depend on timing, topology or the collective library.
__global__ void __launch_bounds__(256)
    sum_shards_kernel(const float* __restrict__ stacked, int nshards, int64_t count, float* __restrict__ out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride) {
    double acc = 0.0;
    for (int r = 0; r < nshards; ++r) acc += static_cast<double>(__ldcs(stacked + r * count + i));
    out[i] = static_cast<float>(acc);
  }
}

// ------------------------------------------------------------------------ diagnostics
//
// Ratio statistics over the counted tokens: sums for the KL estimators k1 = lp_rollout - lp,
// k2 = (lp - lp_rollout)^2 / 2 and k3 = w - 1 - (lp - lp_rollout) (fp64 from the fp32
// inputs, fixed-order per-block partials), min / max of w, max of the deviation |w - 1|
// (w as the loss stage computes it, fp32), and the deviation's exact lower
// median by a three-pass radix select on the deviation's float bits (non-negative floats
// order like their bit patterns; counts are integers, so the result does not depend on
// the order of the atomic adds).
constexpr int kStatThreads = 256;
constexpr int kStatTokens = 4096;  // tokens per block
constexpr int kStatBins = 2048;    // 11 bits per radix pass
constexpr int kStatCtasPerSm = 4;  // resident CTAs per SM of the persistent passes (register-limited)

struct StatPartial {
  double k1, k2, k3;
  float w_min, w_max, dev_max;
  int count;
};

__device__ __forceinline__ float ratio_of(float a, float b) { return ex2_approx((a - b) * kLog2e); }

// e^x - 1 - x.  For |x| < 1/2 the Taylor series x^2 (1/2! + x/3! + ... + x^11/13!)
// (truncation below 1e-14 relative), its first four terms x^2 (1/2 + x/6 + x^2/24 + x^3/120)
// by Horner's rule in fp64 and the rest, x^6 (1/720 + ... + x^7/13!), in fp32: the rest is at
// most |x|^4 / 360 of the whole (1.8e-4 at |x| = 1/2) and carries fp32's ~6e-7 relative
// error of an 8-step Horner sum, so it adds below 1e-10 of relative error.  Outside that
// range expm1(x) - x in fp64.
__device__ __forceinline__ double expm1_minus_x(double x) {
  if (fabs(x) < 0.5) {
    const float xf = static_cast<float>(x);
    float q = 1.0f / 6227020800.0f;  // 1/13!
    q = fmaf(q, xf, 1.0f / 479001600.0f);
    q = fmaf(q, xf, 1.0f / 39916800.0f);
    q = fmaf(q, xf, 1.0f / 3628800.0f);
    q = fmaf(q, xf, 1.0f / 362880.0f);
    q = fmaf(q, xf, 1.0f / 40320.0f);
    q = fmaf(q, xf, 1.0f / 5040.0f);
    q = fmaf(q, xf, 1.0f / 720.0f);
    // p = 1/2 + x (1/6 + x (1/24 + x (1/120 + x q))) with q = 1/720 + x/5040 + ... + x^7/13!
    const double tail = static_cast<double>(q * xf);
    double p = tail + 1.0 / 120.0;
    p = fma(p, x, 1.0 / 24.0);
    p = fma(p, x, 1.0 / 6.0);
    p = fma(p, x, 0.5);
    return p * x * x;
  }
  return expm1(x) - x;
}

// Add 1 to s_hist[bin] for every active lane: one shared-memory atomic per lane; lanes of
// a warp that hit the same bin are serialised by the hardware, which with the clustered
// deviations costs less than grouping the lanes first (__match_any_sync), measured.
__device__ __forceinline__ void hist_add(unsigned* s_hist, unsigned bin, bool active) {
  if (active) atomicAdd(&s_hist[bin], 1u);
}

// A block covers kStatTokens tokens as quads of 4 consecutive tokens, kStatQuads per
// thread, all loaded before any is used (16-byte loads when `vec`: both arrays 16-byte
// aligned; scalar loads at the tail of the array).
constexpr int kStatQuads = kStatTokens / 4 / kStatThreads;

struct StatQuads {
  float a[kStatQuads][4], b[kStatQuads][4];
  bool on[kStatQuads][4];
};

__device__ __forceinline__ void load_stat_quads(const float* __restrict__ lp, const float* __restrict__ lp_roll,
                                                const uint8_t* __restrict__ mask, int64_t n, bool vec, int blk,
                                                StatQuads& q) {
  const int64_t b0 = static_cast<int64_t>(blk) * kStatTokens;
#pragma unroll
  for (int k = 0; k < kStatQuads; ++k) {
    const int64_t t = b0 + 4 * (threadIdx.x + k * kStatThreads);
    if (vec && t + 3 < n) {
      const float4 x = __ldcs(reinterpret_cast<const float4*>(lp + t));
      const float4 y = __ldcs(reinterpret_cast<const float4*>(lp_roll + t));
      q.a[k][0] = x.x, q.a[k][1] = x.y, q.a[k][2] = x.z, q.a[k][3] = x.w;
      q.b[k][0] = y.x, q.b[k][1] = y.y, q.b[k][2] = y.z, q.b[k][3] = y.w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        q.a[k][i] = t + i < n ? __ldcs(lp + t + i) : 0.0f;
        q.b[k][i] = t + i < n ? __ldcs(lp_roll + t + i) : 0.0f;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) q.on[k][i] = t + i < n && (mask == nullptr || mask[t + i] != 0);
  }
}

// Both passes loop over the 4096-token blocks blk = blockIdx.x, blockIdx.x + gridDim.x, ...
// (one block per CTA when the grid covers them all): each block's fp64 partial is computed
// the same way whichever CTA takes it, so the statistics do not depend on the grid, and a
// CTA adds its shared histogram into the global one once, at the end (integer counts).
__global__ void __launch_bounds__(kStatThreads, kStatCtasPerSm)
    ratio_stats_pass0(const float* __restrict__ lp, const float* __restrict__ lp_roll, const uint8_t* __restrict__ mask,
                      int64_t n, bool vec, int nblk, StatPartial* __restrict__ parts, unsigned* __restrict__ hist) {
  __shared__ unsigned s_hist[kStatBins];
  __shared__ StatPartial s_part[kStatThreads / 32];
  for (int b = threadIdx.x; b < kStatBins; b += kStatThreads) s_hist[b] = 0u;
  __syncthreads();
  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
    StatQuads q;
    load_stat_quads(lp, lp_roll, mask, n, vec, blk, q);
    double k1 = 0.0, k2 = 0.0, k3 = 0.0;
    float wmin = INFINITY, wmax = -INFINITY, dmax = 0.0f;
    int cnt = 0;
#pragma unroll
    for (int k = 0; k < kStatQuads; ++k) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool on = q.on[k][i];
        if (on) {
          // the KL estimators in fp64 (k3 cancels to second order); min / max / deviation
          // on the ratio exactly as the loss stage computes it
          const double x = static_cast<double>(q.a[k][i]) - static_cast<double>(q.b[k][i]);
          const float w = ratio_of(q.a[k][i], q.b[k][i]);
          const float dev = fabsf(w - 1.0f);
          k1 -= x;
          k2 += 0.5 * x * x;
          wmin = fminf(wmin, w);
          wmax = fmaxf(wmax, w);
          dmax = fmaxf(dmax, dev);
          ++cnt;
          hist_add(s_hist, __float_as_uint(dev) >> 21, true);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      k1 += __shfl_xor_sync(0xffffffffu, k1, o);
      k2 += __shfl_xor_sync(0xffffffffu, k2, o);
      k3 += __shfl_xor_sync(0xffffffffu, k3, o);
      wmin = fminf(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
      wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
      dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
      cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    }
    if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = StatPartial{k1, k2, k3, wmin, wmax, dmax, cnt};
    __syncthreads();
    if (threadIdx.x == 0) {
      StatPartial acc = s_part[0];
      for (int w = 1; w < kStatThreads / 32; ++w) {
        acc.k1 += s_part[w].k1;
        acc.k2 += s_part[w].k2;
        acc.k3 += s_part[w].k3;
        acc.w_min = fminf(acc.w_min, s_part[w].w_min);
        acc.w_max = fmaxf(acc.w_max, s_part[w].w_max);
        acc.dev_max = fmaxf(acc.dev_max, s_part[w].dev_max);
        acc.count += s_part[w].count;
      }
      parts[blk] = acc;
    }
    __syncthreads();  // s_part is rewritten by the next block
  }
  for (int b = threadIdx.x; b < kStatBins; b += kStatThreads)
    if (s_hist[b]) atomicAdd(&hist[b], s_hist[b]);
}

// Histogram of the next radix digit among the deviations whose higher bits equal `prefix`,
// and half of the k3 sum: in every 4096-token block, each thread's quads k with k % 2 ==
// K3_HALF (the fp64 series is the heaviest arithmetic of the statistics; split evenly over
// the two radix passes, which stream at copy speed with issue slots to spare, it costs every
// SM the same).  The block's half-sum goes to k3_parts[2 blk + K3_HALF], formed the same way
// whichever CTA takes the block (per-thread sums in token order, warp butterfly, warps in
// order), so it does not depend on the grid.
template <int K3_HALF>
__global__ void __launch_bounds__(kStatThreads, kStatCtasPerSm)
    ratio_stats_pass(const float* __restrict__ lp, const float* __restrict__ lp_roll, const uint8_t* __restrict__ mask,
                     int64_t n, bool vec, int nblk, const unsigned* __restrict__ sel, int shift_hi, int shift,
                     unsigned digit_mask, unsigned* __restrict__ hist, double* __restrict__ k3_parts) {
  __shared__ unsigned s_hist[kStatBins];
  __shared__ double s_k3[kStatThreads / 32];
  for (int b = threadIdx.x; b < kStatBins; b += kStatThreads) s_hist[b] = 0u;
  const unsigned prefix = sel[0];
  __syncthreads();
  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
    StatQuads q;
    load_stat_quads(lp, lp_roll, mask, n, vec, blk, q);
    double k3 = 0.0;
#pragma unroll
    for (int k = 0; k < kStatQuads; ++k) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (q.on[k][i]) {
          const unsigned key = __float_as_uint(fabsf(ratio_of(q.a[k][i], q.b[k][i]) - 1.0f));
          if ((key >> shift_hi) == prefix) hist_add(s_hist, (key >> shift) & digit_mask, true);
          if (k % 2 == K3_HALF) k3 += expm1_minus_x(static_cast<double>(q.a[k][i]) - static_cast<double>(q.b[k][i]));
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) k3 += __shfl_xor_sync(0xffffffffu, k3, o);
    if ((threadIdx.x & 31) == 0) s_k3[threadIdx.x >> 5] = k3;
    __syncthreads();
    if (threadIdx.x == 0) {
      double sum = s_k3[0];
      for (int w = 1; w < kStatThreads / 32; ++w) sum += s_k3[w];
      k3_parts[2 * static_cast<int64_t>(blk) + K3_HALF] = sum;
    }
    __syncthreads();  // s_k3 is rewritten by the next block
  }
  for (int b = threadIdx.x; b < kStatBins; b += kStatThreads)
    if (s_hist[b]) atomicAdd(&hist[b], s_hist[b]);
}

// One block: reduce the per-block partials in a fixed order (strided, then a tree) into
// acc, and set the target rank floor((m - 1) / 2) of the lower median.
__global__ void __launch_bounds__(1024)
    ratio_stats_reduce(const StatPartial* __restrict__ parts, int nparts, StatPartial* __restrict__ acc_out,
                       unsigned* __restrict__ sel) {
  __shared__ StatPartial sh[1024];
  StatPartial a{0.0, 0.0, 0.0, INFINITY, -INFINITY, 0.0f, 0};
  for (int b = threadIdx.x; b < nparts; b += blockDim.x) {
    const StatPartial p = parts[b];
    a.k1 += p.k1;
    a.k2 += p.k2;
    a.k3 += p.k3;
    a.w_min = fminf(a.w_min, p.w_min);
    a.w_max = fmaxf(a.w_max, p.w_max);
    a.dev_max = fmaxf(a.dev_max, p.dev_max);
    a.count += p.count;
  }
  sh[threadIdx.x] = a;
  __syncthreads();
  for (int w = blockDim.x >> 1; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      StatPartial& x = sh[threadIdx.x];
      const StatPartial& y = sh[threadIdx.x + w];
      x.k1 += y.k1;
      x.k2 += y.k2;
      x.k3 += y.k3;
      x.w_min = fminf(x.w_min, y.w_min);
      x.w_max = fmaxf(x.w_max, y.w_max);
      x.dev_max = fmaxf(x.dev_max, y.dev_max);
      x.count += y.count;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    *acc_out = sh[0];
    sel[0] = 0u;
    sel[1] = sh[0].count > 0 ? static_cast<unsigned>((sh[0].count - 1) / 2) : 0u;
  }
}

// One block of 1024 threads: find the digit holding rank sel[1] in hist (thread i owns bins
// 2i and 2i + 1; a block-wide exclusive prefix sum gives each bin's first rank), extend the
// prefix, keep the rank within that digit, clear hist for the next pass.  The digit is the
// first bin b with E_b <= rank < E_b + hist[b] (E_b = the counts below b), or the last bin
// when no earlier bin holds the rank.  On the last pass, write the statistics.
constexpr int kSelectThreads = 1024;
static_assert(2 * kSelectThreads >= kStatBins, "two bins per thread");

__global__ void __launch_bounds__(kSelectThreads)
    ratio_stats_select(unsigned* __restrict__ hist, int nbins, int digit_bits, unsigned* __restrict__ sel,
                       const StatPartial* __restrict__ acc_in, int last, double* __restrict__ stats,
                       const double* __restrict__ k3_parts, int nk3) {
  __shared__ unsigned s_warp[kSelectThreads / 32];
  __shared__ double s_k3[kSelectThreads];
  if (last) {  // the k3 sum of all block halves: strided per thread, then a fixed tree
    double a = 0.0;
    for (int b = threadIdx.x; b < nk3; b += kSelectThreads) a += k3_parts[b];
    s_k3[threadIdx.x] = a;
    __syncthreads();
    for (int w = kSelectThreads >> 1; w > 0; w >>= 1) {
      if (threadIdx.x < w) s_k3[threadIdx.x] += s_k3[threadIdx.x + w];
      __syncthreads();
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b0 = 2 * threadIdx.x;
  const unsigned h0 = b0 < nbins ? hist[b0] : 0u;
  const unsigned h1 = b0 + 1 < nbins ? hist[b0 + 1] : 0u;
  const unsigned rank = sel[1];
  const unsigned prefix = sel[0];
  // inclusive scan of h0 + h1 within the warp, then over the warp totals
  unsigned x = h0 + h1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();  // every thread has read sel[] and its bins before anyone writes them
  if (warp == 0) {
    unsigned t = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    s_warp[lane] = t;
  }
  __syncthreads();
  const unsigned e0 = x - (h0 + h1) + (warp > 0 ? s_warp[warp - 1] : 0u);  // E of bin b0
  const unsigned e1 = e0 + h0;                                               // E of bin b0 + 1
  if (b0 < nbins) hist[b0] = 0u;
  if (b0 + 1 < nbins) hist[b0 + 1] = 0u;
  int digit = -1;
  unsigned below = 0u;
  if (b0 < nbins - 1 && rank >= e0 && rank < e0 + h0) {
    digit = b0, below = e0;
  } else if (b0 + 1 < nbins - 1 && rank >= e1 && rank < e1 + h1) {
    digit = b0 + 1, below = e1;
  } else if (b0 == nbins - 1 && rank >= e0) {
    digit = b0, below = e0;
  } else if (b0 + 1 == nbins - 1 && rank >= e1) {
    digit = b0 + 1, below = e1;
  }
  if (digit < 0) return;  // exactly one thread continues
  const unsigned med_bits = (prefix << digit_bits) | static_cast<unsigned>(digit);
  sel[0] = med_bits;
  sel[1] = rank - below;
  if (!last) return;
  const StatPartial acc = *acc_in;
  const double m = acc.count > 0 ? static_cast<double>(acc.count) : 1.0;
  const double med = static_cast<double>(__uint_as_float(med_bits));
  stats[0] = acc.k1 / m;
  stats[1] = acc.k2 / m;
  stats[2] = s_k3[0] / m;
  stats[3] = acc.w_min;
  stats[4] = acc.w_max;
  stats[5] = acc.dev_max;
  stats[6] = med;
  stats[7] = med > 0.0 ? acc.dev_max / med : INFINITY;
  stats[8] = acc.count;
}

// Per response (one warp each): the mean ratio over its counted tokens (0 if none).
__global__ void __launch_bounds__(256)
    response_mean_ratio_kernel(const float* __restrict__ lp, const float* __restrict__ lp_roll,
                               const uint8_t* __restrict__ mask, const int64_t* __restrict__ off, int R,
                               float* __restrict__ out) {
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= R) return;
  double sum = 0.0;
  int c = 0;
  for (int64_t t = off[i] + lane; t < off[i + 1]; t += 32) {
    if (mask != nullptr && mask[t] == 0) continue;
    sum += ratio_of(lp[t], lp_roll[t]);
    ++c;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
  }
  if (lane == 0) out[i] = c > 0 ? static_cast<float>(sum / c) : 0.0f;
}

// Sum of squares of a bf16 (is_bf16) or fp32 array, per-block fp64 partials in a fixed
// order (grid-stride, 8 elements per thread per step), then one block sums the partials.
__global__ void __launch_bounds__(256)
    sumsq_kernel(const void* __restrict__ x, int64_t count, int is_bf16, double* __restrict__ partials) {
  __shared__ double s_w[8];
  double acc = 0.0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride) {
    const float v = is_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(x)[i])
                            : reinterpret_cast<const float*>(x)[i];
    acc += static_cast<double>(v) * v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < 8; ++w) s += s_w[w];
    partials[blockIdx.x] = s;
  }
}

__global__ void sqrt_sum_kernel(const double* __restrict__ partials, int np, double* __restrict__ out) {
  if (threadIdx.x != 0) return;
  double s = 0.0;
  for (int b = 0; b < np; ++b) s += partials[b];
  *out = sqrt(s);
}

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
