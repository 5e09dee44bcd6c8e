// rz_gemm.cuh -- persistent, warp-specialised tcgen05 GEMM engine for sm_100a.
//
//   warp 0      : TMA producer (one elected thread) filling a ring of shared-memory stages
//   warp 1      : TMEM allocator + UMMA issuer (one thread), 128x256x16 bf16 MMAs
//   warps 2..5  : epilogue; warp w reads TMEM lanes 32*(w%4) .. 32*(w%4)+31, so every
//                 epilogue thread owns exactly one output row of the 128-row tile
//
// Tile: BM=128 rows x BN=256 columns, K staged 64 elements (128 bytes) at a time with
// 128-byte swizzle.  The fp32 accumulator lives in TMEM, double-buffered (2 x 256
// columns), so the epilogue of tile i overlaps the MMAs of tile i+1.
//
// Work is a list of units; a unit is one 128-row block times a run of consecutive
// N tiles (the epilogue may carry state across the tiles of a unit, e.g. an online
// log-sum-exp over a vocabulary segment).  Units are dealt to CTAs round-robin
// (unit = blockIdx.x + i*gridDim.x): the schedule never depends on data, uses no
// atomics, and no output element is produced by more than one unit, so results are
// independent of the grid size and of the order in which units run.
//
// Operands: each of A (M x K) and B (N x K) is either K-major (K contiguous; one TMA box
// of 64 x rows) or MN-major (M/N contiguous; boxes of 64 x 64 placed 8 KB apart).  The
// K tail and the M/N tails are zero-filled by TMA out-of-bounds handling.
#pragma once

#include "rz_ptx.cuh"

namespace rz {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;      // bf16 elements per K block (128 bytes)
constexpr int BK_FP8 = 128; // e4m3 elements per K block (128 bytes)
constexpr int kStages = 4;
constexpr int kStageBytesA = BM * BK * 2;  // 16 KB
constexpr int kStageBytesB = BN * BK * 2;  // 32 KB
constexpr int kStageBytes = kStageBytesA + kStageBytesB;
constexpr int kGemmThreads = 192;
constexpr int kTmemCols = 2 * BN;  // two fp32 accumulators of 128 lanes x 256 columns
// Epilogue staging for TMA stores: per epilogue warp, two slots of 32 rows x 64 bytes.
constexpr int kStageSlotBytes = 32 * 64;
constexpr int kEpiWarpStageBytes = 2 * kStageSlotBytes;
constexpr int kEpiStageBytes = 4 * kEpiWarpStageBytes;  // 16 KB
constexpr int kGemmSmemBytes =
    kStages * kStageBytes + kEpiStageBytes + 1024 /*barriers*/ + 1024 /*alignment slack*/;

struct GemmSched {
  int m_blocks;        // number of 128-row blocks
  int n_tiles;         // number of 256-column tiles
  int tiles_per_unit;  // consecutive N tiles processed by one unit
  int units_n;         // ceil(n_tiles / tiles_per_unit)
  int group_m;         // units are ordered in groups of group_m row blocks (L2 locality)
  int group_n;         // with group_m = 1: groups of group_n N-units, each over all row
                       // blocks before the next (group_n >= units_n: no N grouping)
  int num_units;       // m_blocks * units_n
  int num_kb;          // 64-wide K blocks per tile
  int l2_pol_a;        // L2 eviction policy (L2Policy) of the A and B operand loads,
  int l2_pol_b;        // chosen on the host from the operands' sizes and reuse

  // unit index -> (row block, N-unit).  Inside a group of group_m row blocks the row
  // block varies fastest; group_m = 1 gives row-block-major order with N fastest, and
  // with group_n < units_n that order runs group by group over the N-units (the last
  // group holds the remainder).  Either way a bijection onto all units.
  __device__ __forceinline__ void unit_coords(int u, int& mb, int& nu) const {
    if (group_m == 1 && group_n < units_n) {
      const int full = units_n / group_n;   // groups of exactly group_n N-units
      const int span = m_blocks * group_n;  // units per full group
      const int g = u / span;
      if (g < full) {
        const int r = u - g * span;
        mb = r / group_n;
        nu = g * group_n + (r - mb * group_n);
      } else {
        const int rem = units_n - full * group_n;  // > 0 here: u < num_units
        const int r = u - full * span;
        mb = r / rem;
        nu = full * group_n + (r - mb * rem);
      }
      return;
    }
    const int per_group = group_m * units_n;
    const int g = u / per_group;
    const int r = u - g * per_group;
    const int rows_here = min(group_m, m_blocks - g * group_m);
    nu = r / rows_here;
    mb = g * group_m + (r - nu * rows_here);
  }
  __device__ __forceinline__ int unit_tile_begin(int nu) const { return nu * tiles_per_unit; }
  __device__ __forceinline__ int unit_tile_end(int nu) const { return min(n_tiles, (nu + 1) * tiles_per_unit); }
};

// Where the tiles of each operand sit in its tensor map.
//  K-major operand : box (x = k*64, y = row_base + mn0)
//  MN-major operand: boxes (x = mn0 + j*64, y = k_base + k*64), j = 0 .. rows/64-1
struct OperandPos {
  int a_row_base, a_k_base;
  int b_row_base, b_k_base;
};

template <bool MN_MAJOR, int ROWS, int KB_ELEMS = BK>
__device__ __forceinline__ void load_operand(const CUtensorMap* map, uint64_t* bar, uint8_t* dst, int mn0,
                                             int kb, int row_base, int k_base, uint64_t pol) {
  if constexpr (!MN_MAJOR) {
    tma_load_2d(map, bar, dst, kb * KB_ELEMS, row_base + mn0, pol);
  } else {
#pragma unroll
    for (int j = 0; j < ROWS / 64; ++j)
      tma_load_2d(map, bar, dst + j * 8192, mn0 + j * 64, k_base + kb * BK, pol);
  }
}

// Descriptor of one operand stage and the per-UMMA (K = 16) start-address step (>> 4).
//  K-major : rows of 128 B, 8-row groups 1024 B apart (SBO); K step = 32 B.
//  MN-major: 64-element MN atoms 8 KB apart (LBO), 8-row K groups 1024 B apart (SBO);
//            K step = 16 rows = 2048 B.
template <bool MN_MAJOR>
__device__ __forceinline__ uint64_t operand_desc(uint32_t saddr) {
  return MN_MAJOR ? smem_desc_sw128(saddr, 8192, 1024) : smem_desc_sw128(saddr, 16, 1024);
}
template <bool MN_MAJOR>
__host__ __device__ constexpr uint32_t operand_k_step() {
  return MN_MAJOR ? (2048u >> 4) : (32u >> 4);
}

// Per-epilogue-warp staging for TMA stores: two slots of 32 rows x 64 bytes laid out with
// the 64-byte swizzle (16-byte piece q of row r sits at piece q ^ ((r >> 1) & 3)), which
// matches a tensor map with CU_TENSOR_MAP_SWIZZLE_64B and a box of 64 bytes x 32 rows and
// makes the lanes' 16-byte writes bank-conflict free.  Lane 0 issues the store; each
// slot is reused only after the store that last read it has finished reading.
struct WarpStage {
  uint8_t* base;
  int slot;

  // Write this lane's 64-byte row into the next slot and store the slot's 32 x 64-byte
  // box at (x, y) of `map` (reduce-add instead of store when `add` is set).  A box whose
  // first row is at or past `row_limit` lies wholly outside the map and is skipped
  // (uniform across the warp: y is the warp's first row).
  __device__ __forceinline__ void store_rows(const CUtensorMap* map, int lane, const uint4 (&row)[4], int32_t x,
                                             int32_t y, int64_t row_limit, bool add = false) {
    if (y >= row_limit) return;
    uint8_t* buf = base + slot * kStageSlotBytes;
    if (lane == 0) bulk_wait_group_read<1>();  // the store issued from this slot two rounds ago
    __syncwarp();
    uint8_t* r = buf + lane * 64;
    const int sw = (lane >> 1) & 3;
#pragma unroll
    for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(r + ((q ^ sw) << 4)) = row[q];
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (add) tma_reduce_add_2d(map, buf, x, y); else tma_store_2d(map, buf, x, y);
      bulk_commit_group();
    }
    slot ^= 1;
  }
};

// FP8: e4m3 operands (both K-major), kind::f8f6f4, 128-element K blocks; the stage layout
// (128-byte rows, 128-byte swizzle) and the per-instruction 32-byte K step are unchanged.
template <bool A_MN, bool B_MN, class Epi, bool FP8 = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmSched sched, const OperandPos pos, const __grid_constant__ Epi epi,
                   int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* stage_a = smem;
  uint8_t* stage_b = smem + kStages * kStageBytesA;
  uint8_t* epi_stage = smem + kStages * kStageBytes;  // 1024-aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + kEpiStageBytes);
  uint64_t* full = bars;                   // [kStages]  TMA -> MMA
  uint64_t* empty = bars + kStages;        // [kStages]  MMA -> TMA
  uint64_t* acc_full = bars + 2 * kStages; // [2]        MMA -> epilogue
  uint64_t* acc_empty = acc_full + 2;      // [2]        epilogue -> MMA
  uint64_t* mma_done = acc_empty + 2;      // [1]        teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
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
      int issued_phase[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) issued_phase[s] = -1;
      for (int u = blockIdx.x; u < sched.num_units && !aborted; u += gridDim.x) {
        int mb, nu;
        sched.unit_coords(u, mb, nu);
        const int m0 = mb * BM;
        for (int nt = sched.unit_tile_begin(nu); nt < sched.unit_tile_end(nu) && !aborted; ++nt) {
          const int n0 = nt * BN;
          for (int kb = 0; kb < sched.num_kb; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
              aborted = true;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], kStageBytes);
            constexpr int kKb = FP8 ? BK_FP8 : BK;
            load_operand<A_MN, BM, kKb>(&tmA, &full[stage], stage_a + stage * kStageBytesA, m0, kb,
                                        pos.a_row_base, pos.a_k_base, pol_a);
            load_operand<B_MN, BN, kKb>(&tmB, &full[stage], stage_b + stage * kStageBytesB, n0, kb,
                                        pos.b_row_base, pos.b_k_base, pol_b);
            issued_phase[stage] = static_cast<int>(phase);
            if (++stage == kStages) {
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
        for (int s = 0; s < kStages; ++s)
          if (issued_phase[s] >= 0) mbar_wait(&full[s], static_cast<uint32_t>(issued_phase[s]), nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      static_assert(!FP8 || (!A_MN && !B_MN), "e4m3 operands are K-major");
      constexpr uint32_t idesc = FP8 ? idesc_e4m3_f32(BM, BN) : idesc_bf16_f32(BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t it = 0;  // tile counter -> accumulator buffer
      for (int u = blockIdx.x; u < sched.num_units && !aborted; u += gridDim.x) {
        int mb, nu;
        sched.unit_coords(u, mb, nu);
        for (int nt = sched.unit_tile_begin(nu); nt < sched.unit_tile_end(nu) && !aborted; ++nt, ++it) {
          const uint32_t acc = it & 1u;
          if (!mbar_wait(&acc_empty[acc], ((it >> 1) & 1u) ^ 1u, abort_flag)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * BN;
          for (int kb = 0; kb < sched.num_kb; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag)) {
              aborted = true;
              break;
            }
            tc_fence_after();
            const uint64_t a_desc = operand_desc<A_MN>(smem_u32(stage_a + stage * kStageBytesA));
            const uint64_t b_desc = operand_desc<B_MN>(smem_u32(stage_b + stage * kStageBytesB));
#pragma unroll
            for (int k = 0; k < 4; ++k) {  // 4 instructions of 32 bytes of K each
              if constexpr (FP8)
                umma_e4m3(d_tmem, a_desc + k * operand_k_step<A_MN>(), b_desc + k * operand_k_step<B_MN>(), idesc,
                          (kb | k) != 0 ? 1u : 0u);
              else
                umma_bf16(d_tmem, a_desc + k * operand_k_step<A_MN>(), b_desc + k * operand_k_step<B_MN>(), idesc,
                          (kb | k) != 0 ? 1u : 0u);
            }
            umma_commit(&empty[stage]);  // stage reusable once these MMAs have read it
            if (++stage == kStages) {
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
      // every MMA issued above must finish before TMEM is released
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int quad = warp & 3;             // TMEM lane quadrant this warp may access
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    typename Epi::State st;
    WarpStage stage{epi_stage + quad * kEpiWarpStageBytes, 0};
    uint32_t it = 0;
    for (int u = blockIdx.x; u < sched.num_units && !aborted; u += gridDim.x) {
      int mb, nu;
      sched.unit_coords(u, mb, nu);
      epi.begin_unit(st, mb, nu, row_in_tile);
      for (int nt = sched.unit_tile_begin(nu); nt < sched.unit_tile_end(nu); ++nt, ++it) {
        const uint32_t acc = it & 1u;
        // every lane waits, then the warp agrees, so the warp-collective TMEM loads
        // below are never reached by only part of the warp
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], (it >> 1) & 1u, abort_flag));
        if (!ok) {
          aborted = true;
          break;
        }
        tc_fence_after();
        epi.tile(st, lane_base + acc * BN, mb, nt, row_in_tile, lane, stage);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
      }
      if (aborted) break;
      epi.end_unit(st, mb, nu, row_in_tile);
    }
    if (aborted) {
      if (lane == 0) atomicOr(status, kDevWaitTimeout);
      *abort_flag = 1;
    }
    // stores issued from the staging slots complete before the CTA exits
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace rz
