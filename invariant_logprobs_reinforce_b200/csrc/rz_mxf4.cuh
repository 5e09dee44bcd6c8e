// rz_mxf4.cuh -- token logprobs from MXFP4 operands on the block-scaled tensor cores.
//
// The operands are OCP Microscaling MXFP4 (the low-precision LM-head weights of "vLLM says
// aligned kernels make asynchronous RL stable at lag 64" (ainewsbites.com), section "Zero
// mismatch expands to newer models"): every row is cut into 32-element blocks along d; a
// block shares one UE8M0 scale 2^X, X = floor(log2 max|x|) - 2 clamped to [-127, 127] (an
// all-zero block takes X = -127), and each element is the E2M1 value nearest to x / 2^X,
// ties to the even code, saturating at +-6.
//
//   quantize_rows_mxfp4_kernel   bf16 rows -> packed E2M1 codes + tiled UE8M0 scales
//   lmhead_mxf4_lse_kernel       z = H W^T with tcgen05.mma kind::mxf4 (block scales applied
//                                by the tensor cores), the online log-sum-exp of the bf16
//                                forward (same vocabulary segments, same per-row arithmetic)
//
// Layouts in global memory:
//   codes  [rows, d / 2] bytes: element 2j in the low nibble of byte j, 2j + 1 in the high one
//   scales 512-byte atoms, one per (128-row block, 128 columns of d): the scale of row r and
//          32-column block k sits at byte  atom(r / 128, k / 4) * 512 + (r % 32) * 16 +
//          ((r % 128) / 32) * 4 + k % 4,  atoms ordered row block by row block, d / 128 per
//          row block; rows are padded with zero scales to a multiple of 256.  This is the
//          order in which the tensor cores read scale factors from TMEM (one 32-bit column
//          holds one row's four scales; the four 32-row groups of a 128-row block sit in four
//          consecutive columns), so a stage's scales are a plain 1 KB copy per 128 rows.
//
// Kernel: the persistent, warp-specialised shape of the bf16 engine (warp 0 TMA producer,
// warp 1 TMEM allocator + MMA issuer, warps 2..5 epilogue), 128 x 256 tiles, K staged 256
// elements (128 bytes) at a time with 128-byte swizzle, four stages.  Per stage the MMA
// thread copies the stage's scales from shared memory into TMEM (tcgen05.cp, issued before
// and executed in order with the MMAs that read them), then issues four 128x256x64 MMAs.
// The scales need 24 TMEM columns beside the accumulators, so the two accumulator buffers
// overlap by 64 columns (buffer 0 at columns 0..255, buffer 1 at 192..447): the epilogue of
// a tile first copies the 64 shared columns into registers and releases them (ovl_free), so
// the next tile's MMAs can start, and reads the rest while they run.  Every row is still
// processed column by column in the same order (0..255) whichever buffer holds the tile.
#pragma once

#include "rz_simt.cuh"

namespace rz {

constexpr int kMxBlock = 32;          // elements per scale
constexpr int kMxKTile = 256;         // fp4 elements of K per stage (128 bytes per row)
constexpr int kMxStages = 4;
constexpr int kMxStageA = BM * 128;   // 16 KB
constexpr int kMxStageB = BN * 128;   // 32 KB
constexpr int kMxStageSfa = 1024;     // 128 rows x 8 scales
constexpr int kMxStageSfb = 2048;     // 256 rows x 8 scales
constexpr int kMxStageBytes = kMxStageA + kMxStageB + kMxStageSfa + kMxStageSfb;
constexpr int kMxSmemBytes = kMxStages * kMxStageBytes + 1024 /*barriers*/ + 1024 /*alignment slack*/;
constexpr int kMxOverlapCols = 64;                   // columns the two accumulators share
constexpr int kMxAccCol1 = BN - kMxOverlapCols;      // first column of accumulator 1 (192)
constexpr int kMxSfaCol = kMxAccCol1 + BN;           // 448: scales of A (8 columns)
constexpr int kMxSfbCol = kMxSfaCol + 8;             // 456: scales of B (16 columns)
constexpr int kMxTmemCols = 512;
static_assert(kMxSfbCol + 16 <= kMxTmemCols, "scale factors must fit beside the accumulators");
static_assert(kMxSmemBytes <= 232448, "shared memory of one CTA");

// Bytes of the tiled scale array of `rows` rows of d columns (d % 256 == 0).
__host__ __device__ constexpr int64_t mxfp4_scale_bytes(int64_t rows, int d) {
  return ((rows + 255) / 256) * 2 * (d / 128) * 512;
}

// Byte offset of the scale of row r, 32-column block k, in the tiled scale array.
__device__ __forceinline__ int64_t mxfp4_scale_offset(int64_t r, int k, int d) {
  const int64_t atom = (r / 128) * (d / 128) + k / 4;
  const int rr = static_cast<int>(r % 128);
  return atom * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (k % 4);
}

// E2M1 code (sign in bit 3) of y: the nearest of 0, 0.5, 1, 1.5, 2, 3, 4, 6 to |y|, ties to
// the even code, above 5 saturating to 6.  Each comparison is one step up the grid; at a
// midpoint between two codes the even one wins (the strict / non-strict choice per step).
__device__ __forceinline__ uint32_t e2m1_code(float y) {
  const float a = fabsf(y);
  const uint32_t mag = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
  return mag | (signbit(y) ? 8u : 0u);
}

// One thread per (row, 32-element block) of a row-major bf16 [rows, d] array, over rows
// padded to a multiple of 256 (padding rows only write zero scales).  The block exponent is
// read off the bf16 bits of the block maximum: floor(log2 m) = biased exponent - 127 for a
// normal m, so the UE8M0 code X + 127 = max(exponent field - 2, 0), which also gives 0
// (X = -127) for zero and subnormal maxima.  x / 2^X is exact in fp32 here.
__global__ void __launch_bounds__(256)
    quantize_rows_mxfp4_kernel(const __nv_bfloat16* __restrict__ X, int64_t rows, int d, int64_t padded_rows,
                               uint8_t* __restrict__ Q, uint8_t* __restrict__ S) {
  const int nb = d / kMxBlock;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= padded_rows * nb) return;
  const int64_t r = idx / nb;
  const int k = static_cast<int>(idx - r * nb);
  if (r >= rows) {
    S[mxfp4_scale_offset(r, k, d)] = 0;
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(X + r * d + k * kMxBlock);
  uint32_t w[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = __ldg(src + q);
    w[4 * q] = v.x, w[4 * q + 1] = v.y, w[4 * q + 2] = v.z, w[4 * q + 3] = v.w;
  }
  uint32_t amax_bits = 0;  // |x| of a bf16 orders like its bit pattern
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    amax_bits = max(amax_bits, w[i] & 0x7fffu);
    amax_bits = max(amax_bits, (w[i] >> 16) & 0x7fffu);
  }
  const int efield = static_cast<int>(amax_bits >> 7);  // biased exponent of the maximum
  const int code = max(efield - 2, 0);                   // X + 127
  // 2^-X as an fp32 bit pattern: X in [-127, 125], so 2^-X is a normal fp32 (exponent 127 - X)
  const float inv = __uint_as_float(static_cast<uint32_t>(254 - code) << 23);
  uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float lo = __uint_as_float((w[i] & 0xffffu) << 16) * inv;
    const float hi = __uint_as_float(w[i] & 0xffff0000u) * inv;
    const uint32_t byte = e2m1_code(lo) | (e2m1_code(hi) << 4);
    packed[i / 4] |= byte << (8 * (i % 4));
  }
  *reinterpret_cast<uint4*>(Q + r * (d / 2) + k * (kMxBlock / 2)) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  S[mxfp4_scale_offset(r, k, d)] = static_cast<uint8_t>(code);
}

// ---------------------------------------------------------------------------- forward

struct MxfArgs {
  const uint8_t* sfa;  // tiled scales of H
  const uint8_t* sfb;  // tiled scales of W
  int d;
  const int32_t* ids;  // [rows]
  int64_t rows;
  int V;
  int n_tiles;
  float* part_m;
  float* part_s;
  int64_t part_ld;
  float* zy;
};

// The 32 columns of chunk c of the accumulator at `taddr` into v (warp-collective).
__device__ __forceinline__ void tmem_chunk(uint32_t taddr, int c, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld_issue(taddr + c * 32, r);
  tmem_ld_wait(r);
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    lmhead_mxf4_lse_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const GemmSched sched, const __grid_constant__ MxfArgs args, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* stage_a = smem;
  uint8_t* stage_b = stage_a + kMxStages * kMxStageA;
  uint8_t* stage_sfa = stage_b + kMxStages * kMxStageB;
  uint8_t* stage_sfb = stage_sfa + kMxStages * kMxStageSfa;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage_sfb + kMxStages * kMxStageSfb);
  uint64_t* full = bars;                    // [kMxStages]  TMA -> MMA
  uint64_t* empty = bars + kMxStages;       // [kMxStages]  MMA -> TMA
  uint64_t* acc_full = bars + 2 * kMxStages;  // [2]        MMA -> epilogue
  uint64_t* acc_empty = acc_full + 2;       // [2]          epilogue -> MMA (whole buffer read)
  uint64_t* ovl_free = acc_empty + 2;       // [2]          epilogue -> MMA (shared columns read)
  uint64_t* mma_done = ovl_free + 2;        // [1]          teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t sf_row_block_stride = static_cast<int64_t>(args.d / 128) * 512;  // bytes per 128 rows

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);  // one arrival per epilogue warp
      mbar_init(&ovl_free[a], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kMxTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  bool aborted = false;
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint64_t pol_a = make_l2_policy_rt(sched.l2_pol_a);
      const uint64_t pol_b = make_l2_policy_rt(sched.l2_pol_b);
      int issued_phase[kMxStages];
#pragma unroll
      for (int s = 0; s < kMxStages; ++s) issued_phase[s] = -1;
      for (int u = blockIdx.x; u < sched.num_units && !aborted; u += gridDim.x) {
        int mb, nu;
        sched.unit_coords(u, mb, nu);
        for (int nt = sched.unit_tile_begin(nu); nt < sched.unit_tile_end(nu) && !aborted; ++nt) {
          for (int kb = 0; kb < sched.num_kb; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
              aborted = true;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], kMxStageBytes);
            tma_load_2d(&tmA, &full[stage], stage_a + stage * kMxStageA, kb * 128, mb * BM, pol_a);
            tma_load_2d(&tmB, &full[stage], stage_b + stage * kMxStageB, kb * 128, nt * BN, pol_b);
            // scales: atoms 2 kb and 2 kb + 1 of row block mb (A) and of row blocks 2 nt, 2 nt + 1 (B)
            const int64_t koff = static_cast<int64_t>(2 * kb) * 512;
            bulk_load_1d(stage_sfa + stage * kMxStageSfa, args.sfa + mb * sf_row_block_stride + koff, 1024,
                         &full[stage], pol_a);
            uint8_t* sfb = stage_sfb + stage * kMxStageSfb;
            bulk_load_1d(sfb, args.sfb + (2 * nt) * sf_row_block_stride + koff, 1024, &full[stage], pol_b);
            bulk_load_1d(sfb + 1024, args.sfb + (2 * nt + 1) * sf_row_block_stride + koff, 1024, &full[stage],
                         pol_b);
            issued_phase[stage] = static_cast<int>(phase);
            if (++stage == kMxStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      if (aborted) {
        atomicOr(status, kDevWaitTimeout);
        *abort_flag = 1;
        // let copies already in flight land before the CTA's shared memory goes away
        for (int s = 0; s < kMxStages; ++s)
          if (issued_phase[s] >= 0) mbar_wait(&full[s], static_cast<uint32_t>(issued_phase[s]), nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ scale copies + UMMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t it = 0;  // tile counter -> accumulator buffer
      const uint32_t sfa_t = tmem_base + kMxSfaCol;
      const uint32_t sfb_t = tmem_base + kMxSfbCol;
      for (int u = blockIdx.x; u < sched.num_units && !aborted; u += gridDim.x) {
        int mb, nu;
        sched.unit_coords(u, mb, nu);
        for (int nt = sched.unit_tile_begin(nu); nt < sched.unit_tile_end(nu) && !aborted; ++nt, ++it) {
          const uint32_t acc = it & 1u;
          // this buffer fully read by the epilogue of tile it - 2, and the columns it shares
          // with the other buffer read by the epilogue of tile it - 1
          if (!mbar_wait(&acc_empty[acc], ((it >> 1) & 1u) ^ 1u, abort_flag) ||
              (it > 0 && !mbar_wait(&ovl_free[acc ^ 1u], ((it - 1) >> 1) & 1u, abort_flag))) {
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (acc ? kMxAccCol1 : 0);
          for (int kb = 0; kb < sched.num_kb; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag)) {
              aborted = true;
              break;
            }
            tc_fence_after();
            // the stage's scales into TMEM: A atoms (K atom 0, 1) -> columns +0, +4; B atoms
            // (row block h, K atom q) -> columns +8q + 4h
            const uint8_t* sa = stage_sfa + stage * kMxStageSfa;
            const uint8_t* sb = stage_sfb + stage * kMxStageSfb;
            tmem_cp_32x128b_warpx4(sfa_t, smem_desc_rows16(smem_u32(sa)));
            tmem_cp_32x128b_warpx4(sfa_t + 4, smem_desc_rows16(smem_u32(sa + 512)));
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int q = 0; q < 2; ++q)
                tmem_cp_32x128b_warpx4(sfb_t + 8 * q + 4 * h, smem_desc_rows16(smem_u32(sb + h * 1024 + q * 512)));
            const uint64_t a_desc = operand_desc<false>(smem_u32(stage_a + stage * kMxStageA));
            const uint64_t b_desc = operand_desc<false>(smem_u32(stage_b + stage * kMxStageB));
#pragma unroll
            for (int k = 0; k < 4; ++k) {  // K = 64 elements (32 bytes) per instruction
              const uint32_t id = 2u * static_cast<uint32_t>(k & 1);  // byte of the pair of scales
              const uint32_t idesc = idesc_mxf4_f32(BM, BN, id, id);
              umma_mxf4(d_tmem, a_desc + k * operand_k_step<false>(), b_desc + k * operand_k_step<false>(), idesc,
                        (sfa_t + 4u * (k >> 1)) | (id << 30), (sfb_t + 8u * (k >> 1)) | (id << 30),
                        (kb | k) != 0 ? 1u : 0u);
            }
            umma_commit(&empty[stage]);  // stage reusable once these MMAs have read it
            if (++stage == kMxStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (aborted) break;
          umma_commit(&acc_full[acc]);  // accumulator complete
        }
      }
      if (aborted) {
        atomicOr(status, kDevWaitTimeout);
        *abort_flag = 1;
      }
      // every MMA and copy issued above must finish before TMEM is released
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    uint32_t it = 0;
    for (int u = blockIdx.x; u < sched.num_units && !aborted; u += gridDim.x) {
      int mb, nu;
      sched.unit_coords(u, mb, nu);
      const int64_t row = static_cast<int64_t>(mb) * BM + row_in_tile;
      const int y = row < args.rows ? __ldg(args.ids + row) : -1;
      float m = -INFINITY, s = 0.0f;
      for (int nt = sched.unit_tile_begin(nu); nt < sched.unit_tile_end(nu); ++nt, ++it) {
        const uint32_t acc = it & 1u;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], (it >> 1) & 1u, abort_flag));
        if (!ok) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = lane_base + (acc ? kMxAccCol1 : 0);
        // the two chunks this buffer shares with the other one (buffer 0: chunks 6, 7;
        // buffer 1: chunks 0, 1) into registers, then release them to the next tile's MMAs
        const int ov = acc ? 0 : 6;
        float sh[2][32];
        tmem_chunk(taddr, ov, sh[0]);
        tmem_chunk(taddr, ov + 1, sh[1]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ovl_free[acc]);
        // visit chunks c = 0 .. nch - 1 in this order whichever buffer holds the tile: the six
        // unshared chunks stream from TMEM (double-buffered loads), the two shared ones come
        // from the registers
        const int col_base = nt * BN;
        const int nch = min(BN / 32, (args.V - col_base + 31) / 32);  // chunks with a column < V
        auto visit = [&](auto&& fn) {
          if (acc == 0) {
            tmem_for_chunks(taddr, min(nch, 6), fn);
            if (nch > 6) fn(6, sh[0]);
            if (nch > 7) fn(7, sh[1]);
          } else {
            fn(0, sh[0]);
            if (nch > 1) fn(1, sh[1]);
            if (nch > 2) tmem_for_chunks(taddr + 64, nch - 2, [&](int c, float(&v)[32]) { fn(c + 2, v); });
          }
        };
        // one pass over the tile, chunk by chunk in column order: the chunk's maximum (four
        // partial maxima, column j into partial j % 4), the tile's running maximum, the running
        // sum rescaled to it, then the chunk's exponentials as four partial sums added
        // pairwise; every TMEM column is read once.  The raw logit of the sampled token is
        // kept on the way.
        float tmax = -INFINITY, tsum = 0.0f;
        visit([&](int c, float(&v)[32]) {
          const int col0 = col_base + c * 32;
          const bool whole = col0 + 32 <= args.V;
          float cm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          if (whole) {
#pragma unroll
            for (int j = 0; j < 32; ++j) cm[j & 3] = fmaxf(cm[j & 3], v[j]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < args.V) cm[j & 3] = fmaxf(cm[j & 3], v[j]);
          }
          // every visited chunk holds a column < V, so m_new is finite from the first chunk on
          const float m_new = fmaxf(tmax, fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3])));
          const unsigned off = static_cast<unsigned>(y - col0);
          if (off < 32u) {
            float z = v[0];
#pragma unroll
            for (int j = 1; j < 32; ++j) z = (static_cast<unsigned>(j) == off) ? v[j] : z;
            args.zy[row] = z;
          }
          float ts[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          if (whole) {
#pragma unroll
            for (int j = 0; j < 32; ++j) ts[j & 3] += ex2_approx((v[j] - m_new) * kLog2e);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) ts[j & 3] += (col0 + j < args.V) ? ex2_approx((v[j] - m_new) * kLog2e) : 0.0f;
          }
          // first chunk: tmax = -inf, so the old sum (0) is scaled by 2^-inf = 0
          tsum = __fmaf_rn(tsum, ex2_approx(__fmul_rn(tmax - m_new, kLog2e)), (ts[0] + ts[1]) + (ts[2] + ts[3]));
          tmax = m_new;
        });
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
        lse_fold(m, s, tmax, tsum);
      }
      if (aborted) break;
      if (row < args.rows) {
        args.part_m[static_cast<int64_t>(nu) * args.part_ld + row] = m;
        args.part_s[static_cast<int64_t>(nu) * args.part_ld + row] = s;
      }
    }
    if (aborted) {
      if (lane == 0) atomicOr(status, kDevWaitTimeout);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kMxTmemCols);
  }
}

}  // namespace rz
