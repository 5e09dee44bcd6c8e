// rz_api.cu -- the C ABI declared in include/rz.h: argument checks, workspace carving,
// TMA descriptor creation and the launch sequence of each entry point.
//
// Launch sequence of rz_loss_fwd_bwd (all on the caller's stream, no host sync):
//   1. loss setup : group sums, per-response coefficients -A_i/(N L_i), block starts
//   2. for each chunk of 16384 tokens, in order:
//        forward  : fused LM head + online log-sum-exp per (128-row block, 2048-column
//                   vocabulary segment), keeping e = exp(z - tile max) (fp16); merge -> lp, lse
//        kappa    : per-token ratio and kappa, per-4096-token loss partials
//        dZ       : kappa (onehot - e exp(tile max - lse)) as bf16, in place of e
//        backward : dH rows = dZ W;  dW (+)= dZ^T H
//   3. loss       : fixed-order sum of the partials
// With the sequence gate a forward pass over every chunk runs first (the gate needs all
// logprobs); rz_loss_fwd_bwd_streamed copies each chunk's rows of H from host memory on a
// copy stream one chunk ahead.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/rz.h"
#include "rz_mxf4.cuh"

namespace rz {
namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool shape_ok(int32_t d, int32_t V) { return d >= 64 && d <= 32768 && d % 64 == 0 && V >= 1; }

int num_segments(int32_t V) { return static_cast<int>(ceil_div(V, kSegWidth)); }
int num_vocab_tiles(int32_t V) { return static_cast<int>(ceil_div(V, BN)); }

// A forward-only call whose (row block, segment) units would leave most SMs idle (a decode
// step of a few rows) runs one unit per 256-column tile instead and the merge folds each
// segment's tiles in order (merge_lse_kernel): the same bits, with up to eight times the
// units.  The threshold is a constant (two units per SM of a 148-SM B200), not a query of
// the device, so workspace sizes do not depend on the device.
constexpr int64_t kTileUnitsBelow = 296;
bool tile_units(int64_t rows, int32_t V) { return ceil_div(rows, BM) * num_segments(V) < kTileUnitsBelow; }

int64_t padded_vocab(int32_t V) { return align_up(static_cast<size_t>(V), 8); }

int kappa_blocks(int64_t n) { return static_cast<int>(ceil_div(n, static_cast<int64_t>(kKappaBlockTokens))); }

// Rows processed together by the loss path (one backward chunk).
int64_t chunk_capacity(int64_t n) { return std::min<int64_t>(align_up(n, BM), kChunkTokens); }

// Workspace layout (byte offsets from the workspace base, each 256-byte aligned).
//  forward only  : status | part_m [S][n] | part_s [S][n] | zy [n]
//  loss path     : status | part_m [S][C] | part_s [S][C] | zy [C] | lp, lse, kappa [n]
//                  | coef [R] | gsum [G] | gcnt [G] | bsum, bfirst [blocks] | tile_max [C][tiles]
//                  | e / dZ buffer [C][V rounded up to 8] (16-bit)
//  loss stage    : status | lp.. as above without the forward and backward pieces
struct Layout {
  size_t status = 0;
  size_t part_m = 0, part_s = 0, zy = 0;
  int64_t part_ld = 0;
  size_t lp = 0, lse = 0, kappa = 0;
  size_t coef = 0, gsum = 0, gcnt = 0, bsum = 0, bfirst = 0, counted = 0;
  size_t tile_max = 0, dz = 0;
  size_t total = 0;
};

enum class Path { Forward, Loss, LossStage };

Layout make_layout(int64_t n, int32_t R, int32_t G, int32_t V, Path path) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, kAlign);
    return at;
  };
  L.status = take(16);
  if (path != Path::LossStage) {
    // partial columns: one per segment, or one per tile for a forward call of few row blocks
    const int S = (path == Path::Forward && tile_units(n, V)) ? num_vocab_tiles(V) : num_segments(V);
    L.part_ld = path == Path::Forward ? n : chunk_capacity(n);
    L.part_m = take(sizeof(float) * static_cast<size_t>(S) * L.part_ld);
    L.part_s = take(sizeof(float) * static_cast<size_t>(S) * L.part_ld);
    L.zy = take(sizeof(float) * L.part_ld);
  }
  if (path != Path::Forward) {
    L.lp = take(sizeof(float) * n);
    L.lse = take(sizeof(float) * n);
    L.kappa = take(sizeof(float) * n);
    L.coef = take(sizeof(float) * R);
    L.gsum = take(sizeof(double) * G);
    L.gcnt = take(sizeof(int) * G);
    L.bsum = take(sizeof(double) * kappa_blocks(n));
    L.bfirst = take(sizeof(int) * kappa_blocks(n));
    L.counted = take(sizeof(int) * R);
  }
  if (path == Path::Loss) {
    const int64_t C = chunk_capacity(n);
    L.tile_max = take(sizeof(float) * static_cast<size_t>(C) * num_vocab_tiles(V));
    L.dz = take(sizeof(uint16_t) * static_cast<size_t>(C) * padded_vocab(V));
  }
  L.total = off;
  return L;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// ---------------------------------------------------------------- driver entry point

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D tensor map over a row-major [outer, inner] array with the given row stride (bytes),
// box {box_inner, box_outer}, zero fill out of bounds.
bool make_map(CUtensorMap* m, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Operand load map: bf16, box {64, box_outer}, 128-byte swizzle (the UMMA stage layout).
bool make_operand_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                      uint32_t box_outer) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, inner, outer, row_stride_bytes, 64, box_outer,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// Epilogue store map: 32 rows x 64 bytes with the 64-byte swizzle of the staging slots.
bool make_store_map(CUtensorMap* m, CUtensorMapDataType dtype, uint32_t elem_bytes, const void* base,
                    uint64_t inner, uint64_t outer, uint64_t row_stride_bytes) {
  return make_map(m, dtype, base, inner, outer, row_stride_bytes, 64 / elem_bytes, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

// ---------------------------------------------------------------- launch recorder

// Optional per-launch CUDA events (rz_loss_fwd_bwd_timed): an event pair around each
// kernel launch, in launch order, with the kernel kind of each launch.
struct Recorder {
  cudaEvent_t* events;  // [2 * cap]
  int32_t* kinds;       // [cap]
  int32_t cap;
  int32_t count;
  bool open;
};

void rec_begin(Recorder* r, int kind, cudaStream_t s) {
  if (r == nullptr) return;
  r->open = r->count < r->cap;
  if (!r->open) return;
  r->kinds[r->count] = kind;
  cudaEventRecord(r->events[2 * r->count], s);
}

void rec_end(Recorder* r, cudaStream_t s) {
  if (r == nullptr || !r->open) return;
  cudaEventRecord(r->events[2 * r->count + 1], s);
  ++r->count;
  r->open = false;
}

// ---------------------------------------------------------------- launches

int sm_count() {
  static std::atomic<int> cache[kMaxDevices];  // zero-initialised (static storage)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDevices) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDevices) cache[dev].store(sms, std::memory_order_relaxed);
  return sms;
}

// The engine's dynamic shared memory is above the 48 KB default, so each kernel
// instantiation needs its limit raised once per device; the devices done are kept as bits
// of a per-instantiation word (setting it twice from racing threads is harmless).
template <bool A_MN, bool B_MN, class Epi, bool FP8>
cudaError_t ensure_gemm_smem_attr() {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  err = cudaFuncSetAttribute(gemm_tc_kernel<A_MN, B_MN, Epi, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemmSmemBytes);
  if (err == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_acq_rel);
  return err;
}

template <bool A_MN, bool B_MN, class Epi, bool FP8 = false>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const GemmSched& s, const OperandPos& p,
                        const Epi& e, int* status, cudaStream_t stream) {
  auto kernel = gemm_tc_kernel<A_MN, B_MN, Epi, FP8>;
  cudaError_t err = ensure_gemm_smem_attr<A_MN, B_MN, Epi, FP8>();
  if (err != cudaSuccess) return err;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int grid = std::max(1, std::min(s.num_units, sms));
  kernel<<<grid, kGemmThreads, kGemmSmemBytes, stream>>>(a, b, s, p, e, status);
  return cudaGetLastError();
}

// L2 eviction policies of the operand loads, from the operands' sizes and reuse (L2 126 MB):
//  - an operand re-read by every wave of tiles stays (evict-last) while it fits in what
//    the streams leave of L2: the forward's group of H row blocks, the columns of dW's
//    chunk of H that one group of output tiles reads;
//  - a streamed operand read by the output tiles of its row block side by side goes first
//    (evict-first) while those tiles are few (at most 12; larger d runs its tiles in groups
//    of at most 12, see backward_group_n): dZ in dH and dW; with more consumers its lines
//    must survive until the last of them has read them;
//  - W in the forward-only call goes first (nothing else streams through L2 there).
constexpr uint64_t kL2KeepBytes = 96ull << 20;
constexpr int kFewConsumerTiles = 12;

int keep_if_fits(uint64_t bytes) { return bytes <= kL2KeepBytes ? kL2EvictLast : kL2Normal; }

// Row blocks per L2 group of the forward: the largest power of two up to 32 whose H rows
// (128 per block, d elements of elem_bytes) take at most 24 MB, so the group stays in L2
// beside the W tiles in flight and the stored exponentials (32 at d = 2560, 8 at d = 7168).
// It only orders the units; no row's arithmetic depends on it.
int forward_group_m(int32_t d, int elem_bytes) {
  const uint64_t block_bytes = static_cast<uint64_t>(BM) * d * elem_bytes;
  int g = 32;
  while (g > 1 && g * block_bytes > (24ull << 20)) g >>= 1;
  return g;
}
int first_if_few(int consumer_tiles) { return consumer_tiles <= kFewConsumerTiles ? kL2EvictFirst : kL2Normal; }

// dH with more than kFewConsumerTiles output tiles per row block (d > 3072) runs its N tiles
// in balanced groups of at most that many: a wave then streams only its group's slice of
// W, and a dZ row block has only the group's tiles as consumers, at the price of reading dZ
// once per group (dW groups by the size of its slice of H, dw_group_n).
int backward_group_n(int n_tiles) {
  if (n_tiles <= kFewConsumerTiles) return n_tiles;
  const int groups = (n_tiles + kFewConsumerTiles - 1) / kFewConsumerTiles;
  return (n_tiles + groups - 1) / groups;
}

// dW's column tiles run in balanced groups whose slice of the chunk's H (kept in L2 with
// evict-last while the group's waves stream dZ past it) takes at most 48 MB, and at most
// kFewConsumerTiles tiles: at d = 2560 and 16384-row chunks two groups of 5 (42 MB each)
// instead of one of 10 (84 MB), at the price of reading dZ once per group.  Measured on one
// box: dW 233 vs 240-243 ms per step, the step 767-768 vs 778-783 ms (less DRAM traffic, so a
// higher clock under the power cap).
constexpr uint64_t kDwSliceBytes = 48ull << 20;
int dw_group_n(int n_tiles, int64_t rows) {
  const uint64_t tile_bytes = static_cast<uint64_t>(std::max<int64_t>(rows, 1)) * BN * 2;
  const int cap = static_cast<int>(
      std::min<uint64_t>(kFewConsumerTiles, std::max<uint64_t>(1, kDwSliceBytes / tile_bytes)));
  const int groups = (n_tiles + cap - 1) / cap;
  return (n_tiles + groups - 1) / groups;
}

GemmSched make_sched(int64_t m_rows, int64_t n_cols, int tiles_per_unit, int group_m, int64_t k) {
  GemmSched s;
  s.l2_pol_a = kL2Normal;
  s.l2_pol_b = kL2Normal;
  s.m_blocks = static_cast<int>(ceil_div(m_rows, BM));
  s.n_tiles = static_cast<int>(ceil_div(n_cols, BN));
  s.tiles_per_unit = tiles_per_unit;
  s.units_n = static_cast<int>(ceil_div(s.n_tiles, tiles_per_unit));
  s.group_m = std::max(1, std::min(group_m, s.m_blocks));
  s.group_n = s.units_n;
  s.num_units = s.m_blocks * s.units_n;
  s.num_kb = static_cast<int>(ceil_div(k, BK));
  return s;
}

// Forward over rows [r0, r0 + rows): the fused LM head + online log-sum-exp kernel writes
// per-segment partials (row stride L.part_ld, rows launch-relative); the merge writes lp
// and lse (nullable) for those rows.  With store_p the kernel also writes the fp16
// exponentials e = exp(z - tile_max) and the tile maxima for the backward.
rz_status run_forward(const rz_bf16* H, const rz_bf16* W, const int32_t* ids, int64_t r0, int64_t rows, int32_t d,
                      int32_t V, float* lp, float* lse, void* ws, const Layout& L, bool store_p, cudaStream_t stream,
                      Recorder* rec, bool allow_tile_units = false) {
  int* status = at<int>(ws, L.status);
  CUtensorMap mH, mW;
  // rows past the range read as zeros, so no other rows' data enters the launch
  if (!make_operand_map(&mH, H, d, r0 + rows, static_cast<uint64_t>(d) * 2, BM)) return RZ_ERR_CUDA;
  if (!make_operand_map(&mW, W, d, V, static_cast<uint64_t>(d) * 2, BN)) return RZ_ERR_CUDA;
  const bool per_tile = allow_tile_units && !store_p && tile_units(rows, V);
  GemmSched s = make_sched(rows, V, per_tile ? 1 : kSegTiles, forward_group_m(d, 2), d);
  s.l2_pol_a = keep_if_fits(static_cast<uint64_t>(std::min<int64_t>(s.group_m * BM, rows)) * d * 2);
  s.l2_pol_b = store_p ? kL2Normal : kL2EvictFirst;
  const OperandPos pos{static_cast<int>(r0), 0, 0, 0};
  float* part_m = at<float>(ws, L.part_m);
  float* part_s = at<float>(ws, L.part_s);
  float* zy = at<float>(ws, L.zy);
  rec_begin(rec, RZ_KERNEL_LMHEAD_LSE, stream);
  if (store_p) {
    EpiLse<true> e;
    if (!make_store_map(&e.p_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, at<uint16_t>(ws, L.dz), V, rows,
                        static_cast<uint64_t>(padded_vocab(V)) * 2))
      return RZ_ERR_CUDA;
    e.ids = ids + r0;
    e.rows = rows;
    e.V = V;
    e.n_tiles = num_vocab_tiles(V);
    e.part_m = part_m;
    e.part_s = part_s;
    e.part_ld = L.part_ld;
    e.zy = zy;
    e.tile_max = at<float>(ws, L.tile_max);
    e.row_scale = nullptr;
    e.col_scale = nullptr;
    e.col_scale_vec = 0;
    if (launch_gemm<false, false>(mH, mW, s, pos, e, status, stream) != cudaSuccess) return RZ_ERR_CUDA;
  } else {
    EpiLse<false> e;
    std::memset(&e.p_map, 0, sizeof(e.p_map));
    e.ids = ids + r0;
    e.rows = rows;
    e.V = V;
    e.n_tiles = num_vocab_tiles(V);
    e.part_m = part_m;
    e.part_s = part_s;
    e.part_ld = L.part_ld;
    e.zy = zy;
    e.tile_max = nullptr;
    e.row_scale = nullptr;
    e.col_scale = nullptr;
    e.col_scale_vec = 0;
    if (launch_gemm<false, false>(mH, mW, s, pos, e, status, stream) != cudaSuccess) return RZ_ERR_CUDA;
  }
  rec_end(rec, stream);
  const int threads = 256;
  rec_begin(rec, RZ_KERNEL_MERGE_LSE, stream);
  merge_lse_kernel<<<static_cast<unsigned>(ceil_div(rows, threads)), threads, 0, stream>>>(
      part_m, part_s, L.part_ld, zy, ids + r0, rows, V, num_segments(V), lp + r0, lse ? lse + r0 : nullptr, status,
      per_tile ? num_vocab_tiles(V) : 0);
  if (cudaGetLastError() != cudaSuccess) return RZ_ERR_CUDA;
  rec_end(rec, stream);
  return RZ_OK;
}

// Forward with scaled e4m3 operands (kind::f8f6f4, 128-element K blocks): the same
// epilogue and merge as run_forward, with the logits rescaled per row and column.
rz_status run_forward_fp8(const uint8_t* H8, const float* hs, const uint8_t* W8, const float* wsc,
                          const int32_t* ids, int64_t n, int32_t d, int32_t V, float* lp, float* lse, void* ws,
                          const Layout& L, cudaStream_t stream) {
  int* status = at<int>(ws, L.status);
  CUtensorMap mH, mW;
  if (!make_map(&mH, CU_TENSOR_MAP_DATA_TYPE_UINT8, H8, d, n, static_cast<uint64_t>(d), BK_FP8, BM,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return RZ_ERR_CUDA;
  if (!make_map(&mW, CU_TENSOR_MAP_DATA_TYPE_UINT8, W8, d, V, static_cast<uint64_t>(d), BK_FP8, BN,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return RZ_ERR_CUDA;
  GemmSched s = make_sched(n, V, kSegTiles, forward_group_m(d, 1), d);
  s.num_kb = static_cast<int>(ceil_div(d, BK_FP8));
  s.l2_pol_a = keep_if_fits(static_cast<uint64_t>(std::min<int64_t>(s.group_m * BM, n)) * d);  // e4m3
  s.l2_pol_b = kL2EvictFirst;
  const OperandPos pos{0, 0, 0, 0};
  EpiLse<false, true> e;
  std::memset(&e.p_map, 0, sizeof(e.p_map));
  e.ids = ids;
  e.rows = n;
  e.V = V;
  e.n_tiles = num_vocab_tiles(V);
  e.part_m = at<float>(ws, L.part_m);
  e.part_s = at<float>(ws, L.part_s);
  e.part_ld = L.part_ld;
  e.zy = at<float>(ws, L.zy);
  e.tile_max = nullptr;
  e.row_scale = hs;
  e.col_scale = wsc;
  e.col_scale_vec = aligned(wsc, 16) ? 1 : 0;
  if (launch_gemm<false, false, EpiLse<false, true>, true>(mH, mW, s, pos, e, status, stream) != cudaSuccess)
    return RZ_ERR_CUDA;
  merge_lse_kernel<<<static_cast<unsigned>(ceil_div(n, 256)), 256, 0, stream>>>(
      e.part_m, e.part_s, L.part_ld, e.zy, ids, n, V, num_segments(V), lp, lse, status);
  return cudaGetLastError() == cudaSuccess ? RZ_OK : RZ_ERR_CUDA;
}

// Forward from MXFP4 operands (kind::mxf4, block scales applied by the tensor cores): the
// same vocabulary segments, per-row log-sum-exp arithmetic and merge as run_forward.
rz_status run_forward_mxfp4(const uint8_t* H4, const uint8_t* hs, const uint8_t* W4, const uint8_t* wsc,
                            const int32_t* ids, int64_t n, int32_t d, int32_t V, float* lp, float* lse, void* ws,
                            const Layout& L, cudaStream_t stream) {
  int* status = at<int>(ws, L.status);
  CUtensorMap mH, mW;
  // packed codes: d / 2 bytes per row, boxes of 128 bytes (256 elements) x rows
  if (!make_map(&mH, CU_TENSOR_MAP_DATA_TYPE_UINT8, H4, d / 2, n, static_cast<uint64_t>(d / 2), 128, BM,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return RZ_ERR_CUDA;
  if (!make_map(&mW, CU_TENSOR_MAP_DATA_TYPE_UINT8, W4, d / 2, V, static_cast<uint64_t>(d / 2), 128, BN,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return RZ_ERR_CUDA;
  GemmSched s = make_sched(n, V, kSegTiles, forward_group_m(d / 2, 1), d);
  s.num_kb = static_cast<int>(ceil_div(d, kMxKTile));
  s.l2_pol_a = keep_if_fits(static_cast<uint64_t>(std::min<int64_t>(s.group_m * BM, n)) * (d / 2));
  s.l2_pol_b = kL2EvictFirst;
  MxfArgs a;
  a.sfa = hs;
  a.sfb = wsc;
  a.d = d;
  a.ids = ids;
  a.rows = n;
  a.V = V;
  a.n_tiles = num_vocab_tiles(V);
  a.part_m = at<float>(ws, L.part_m);
  a.part_s = at<float>(ws, L.part_s);
  a.part_ld = L.part_ld;
  a.zy = at<float>(ws, L.zy);
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RZ_ERR_CUDA;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit == 0 || !(attr_done.load(std::memory_order_acquire) & bit)) {
    if (cudaFuncSetAttribute(lmhead_mxf4_lse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMxSmemBytes) !=
        cudaSuccess)
      return RZ_ERR_CUDA;
    if (bit != 0) attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  const int sms = sm_count();
  if (sms <= 0) return RZ_ERR_CUDA;
  lmhead_mxf4_lse_kernel<<<std::max(1, std::min(s.num_units, sms)), kGemmThreads, kMxSmemBytes, stream>>>(mH, mW, s,
                                                                                                        a, status);
  if (cudaGetLastError() != cudaSuccess) return RZ_ERR_CUDA;
  merge_lse_kernel<<<static_cast<unsigned>(ceil_div(n, 256)), 256, 0, stream>>>(
      a.part_m, a.part_s, L.part_ld, a.zy, ids, n, V, num_segments(V), lp, lse, status);
  return cudaGetLastError() == cudaSuccess ? RZ_OK : RZ_ERR_CUDA;
}

// Loss-stage options after defaults: no cap (+inf), no gate, no mask, N = n_resp.
struct LossOpts {
  float clip_max = INFINITY;
  bool gate = false;
  double gate_lo = 0.0, gate_hi = INFINITY;
  const uint8_t* mask = nullptr;
  double N = 0.0;
};

bool resolve_options(const rz_loss_options* o, int32_t n_resp, LossOpts* out) {
  LossOpts r;
  r.N = static_cast<double>(n_resp);
  if (o != nullptr) {
    if (o->flags & ~(RZ_LOSS_CLIP_IS | RZ_LOSS_SEQ_GATE | RZ_LOSS_TOKEN_MASK)) return false;
    if (o->flags & RZ_LOSS_CLIP_IS) {
      if (!(o->clip_max > 0.0f)) return false;
      r.clip_max = o->clip_max;
    }
    if (o->flags & RZ_LOSS_SEQ_GATE) {
      if (!(o->gate_lo <= o->gate_hi)) return false;
      r.gate = true;
      r.gate_lo = o->gate_lo;
      r.gate_hi = o->gate_hi;
    }
    if (o->flags & RZ_LOSS_TOKEN_MASK) {
      if (o->token_mask == nullptr || !aligned(o->token_mask, 4)) return false;
      r.mask = o->token_mask;
    }
    if (o->n_resp_total < 0) return false;
    if (o->n_resp_total > 0) r.N = static_cast<double>(o->n_resp_total);
  }
  *out = r;
  return true;
}

// Loss stage, part 1: checks, group sums, coef_i = -A_i/(N L_i) (L_i = counted tokens
// under a mask), first response per block.
rz_status run_loss_setup(const float* rewards, const int64_t* off, const int32_t* gid, int64_t n, int32_t R,
                         int32_t G, const LossOpts& opt, void* ws, const Layout& L, cudaStream_t stream,
                         Recorder* rec) {
  int* status = at<int>(ws, L.status);
  int* flags = status + 1;  // unsorted flag, then the tickets; cleared with the status word
  int* counted = nullptr;
  rec_begin(rec, RZ_KERNEL_RESPONSE_COEF, stream);
  if (opt.mask != nullptr) {
    counted = at<int>(ws, L.counted);
    masked_count_kernel<<<static_cast<unsigned>(ceil_div(R, 8)), 256, 0, stream>>>(opt.mask, off, R, counted);
    if (cudaGetLastError() != cudaSuccess) return RZ_ERR_CUDA;
  }
  const int nb = kappa_blocks(n);
  const unsigned grid = static_cast<unsigned>(ceil_div(R, kSetupThreads));
  loss_setup_kernel<<<grid, kSetupThreads, 0, stream>>>(rewards, off, gid, R, G, n, opt.N, counted,
                                                        at<double>(ws, L.gsum), at<int>(ws, L.gcnt),
                                                        at<float>(ws, L.coef), nb, at<int>(ws, L.bfirst), flags,
                                                        flags + 1, status);
  if (cudaGetLastError() != cudaSuccess) return RZ_ERR_CUDA;
  rec_end(rec, stream);
  return RZ_OK;
}

// Sequence gate: zero the coefficient of every response whose geometric-mean ratio lies
// outside [gate_lo, gate_hi] (needs lp of all tokens).
rz_status run_gate(const float* lp, const float* lp_roll, const int64_t* off, int32_t R, const LossOpts& opt,
                   void* ws, const Layout& L, cudaStream_t stream) {
  gate_kernel<<<static_cast<unsigned>(ceil_div(R, 8)), 256, 0, stream>>>(lp, lp_roll, opt.mask, off, R, opt.gate_lo,
                                                                      opt.gate_hi, at<float>(ws, L.coef));
  return cudaGetLastError() == cudaSuccess ? RZ_OK : RZ_ERR_CUDA;
}

// The kappa kernels' dynamic shared memory (bulk-copy stages) exceeds the default limit:
// raised once per device and variant (devices done kept as bits, as for the GEMM kernels).
cudaError_t ensure_kappa_smem_attr(bool masked, bool clipped, const void* kernel, int smem) {
  static std::atomic<uint64_t> done[4];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::atomic<uint64_t>& word = done[(masked ? 2 : 0) + (clipped ? 1 : 0)];
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit != 0 && (word.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err == cudaSuccess && bit != 0) word.fetch_or(bit, std::memory_order_acq_rel);
  return err;
}

// Loss stage, part 2: kappa and ratio for the 4096-token blocks [blk0, blk0 + nblk); the
// block that finishes last of all the call's blocks writes the loss.  after_setup: the
// kernel directly before this one on the stream is the setup kernel, so this one is
// launched as its programmatic dependent (its lp / lp_rollout loads overlap the setup; it
// waits for the setup's results before reading them).  Only then: lp may come from the
// kernel before, which a programmatic launch would not wait for.
rz_status run_kappa(const float* lp, const float* lp_roll, const int64_t* off, int64_t n, int32_t R, int blk0,
                    int nblk, const LossOpts& opt, float* kappa, float* w_out, float* loss, void* ws, const Layout& L,
                    cudaStream_t stream, Recorder* rec, bool after_setup = false) {
  // whole blocks are bulk-copied into shared memory and kappa / w are stored four at a
  // time: both need 16-byte aligned arrays (a 4096-token block then starts 16-byte aligned)
  const int vec_ok = aligned(lp, 16) && aligned(lp_roll, 16) && aligned(kappa, 16) &&
                     (w_out == nullptr || aligned(w_out, 16)) && (opt.mask == nullptr || aligned(opt.mask, 16));
  rec_begin(rec, RZ_KERNEL_TOKEN_KAPPA, stream);
  // min(w, +inf) = w, so the unclipped variant gives the same bits as a clip at +inf would
  const bool masked = opt.mask != nullptr, clipped = !std::isinf(opt.clip_max);
  auto kernel = masked ? (clipped ? token_kappa_kernel<true, true> : token_kappa_kernel<true, false>)
                       : (clipped ? token_kappa_kernel<false, true> : token_kappa_kernel<false, false>);
  const int smem = masked ? KappaSmem<true>::kBytes : KappaSmem<false>::kBytes;
  if (ensure_kappa_smem_attr(masked, clipped, reinterpret_cast<const void*>(kernel), smem) != cudaSuccess)
    return RZ_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return RZ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  const int ctas = masked ? KappaSmem<true>::kCtasPerSm : KappaSmem<false>::kCtasPerSm;
  cfg.gridDim = dim3(static_cast<unsigned>(std::max(1, std::min(nblk, ctas * sms))));
  cfg.blockDim = dim3(kKappaThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (after_setup && rec == nullptr) ? 1 : 0;  // a recorded event in between would end the overlap
  const float* coef = at<float>(ws, L.coef);
  const int* bfirst = at<int>(ws, L.bfirst);
  int* status = at<int>(ws, L.status);
  if (cudaLaunchKernelEx(&cfg, kernel, lp, lp_roll, off, R, coef, bfirst, n, blk0, nblk, vec_ok, opt.mask,
                         opt.clip_max, kappa, w_out, at<double>(ws, L.bsum), kappa_blocks(n), status + 3, loss,
                         status) != cudaSuccess)
    return RZ_ERR_CUDA;
  rec_end(rec, stream);
  return RZ_OK;
}

rz_status run_segment_loss(const float* lp, const float* lp_roll, const float* rewards, const int64_t* off,
                           const int32_t* gid, int64_t n, int32_t R, int32_t G, const LossOpts& opt, float* loss,
                           float* kappa, float* w_out, void* ws, const Layout& L, cudaStream_t stream,
                           Recorder* rec) {
  rz_status r = run_loss_setup(rewards, off, gid, n, R, G, opt, ws, L, stream, rec);
  if (r != RZ_OK) return r;
  if (opt.gate) {
    r = run_gate(lp, lp_roll, off, R, opt, ws, L, stream);
    if (r != RZ_OK) return r;
  }
  return run_kappa(lp, lp_roll, off, n, R, 0, kappa_blocks(n), opt, kappa, w_out, loss, ws, L, stream, rec,
                   /*after_setup=*/!opt.gate);
}

// A non-blocking stream per device for device-to-host copies of results, created on
// first use (separate from the host-to-device stream, so both copy directions overlap).
cudaStream_t d2h_stream_for_current_device() {
  static std::mutex mu;
  static cudaStream_t streams[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (streams[dev] == nullptr && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess)
    streams[dev] = nullptr;
  return streams[dev];
}

// Results copied to host memory as they are produced (rz_loss_fwd_bwd_host_io): each
// chunk's dH rows right after that chunk's dH contraction, dW after the last chunk's dW
// contraction, on the device-to-host stream, so the copies of chunk c run while chunk
// c + 1 computes.  finish() makes the compute stream wait for every copy, so the call's
// work on that stream completes only once the host buffers hold the results.
struct HostExport {
  rz_bf16* dH_host;  // nullable
  float* dW_host;    // nullable
  cudaStream_t copy = nullptr;
  cudaEvent_t ev = nullptr;

  HostExport(rz_bf16* dh, float* dw) : dH_host(dh), dW_host(dw) {}
  HostExport(const HostExport&) = delete;
  HostExport& operator=(const HostExport&) = delete;
  ~HostExport() {
    if (ev != nullptr) cudaEventDestroy(ev);  // released once its pending records complete
  }

  rz_status start() {
    copy = d2h_stream_for_current_device();
    if (copy == nullptr) return RZ_ERR_CUDA;
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) {
      ev = nullptr;
      return RZ_ERR_CUDA;
    }
    return RZ_OK;
  }

  // Copy `bytes` from device `src` to host `dst` once the work enqueued on `st` so far is done.
  rz_status copy_after(cudaStream_t st, void* dst, const void* src, size_t bytes) {
    if (cudaEventRecord(ev, st) != cudaSuccess || cudaStreamWaitEvent(copy, ev, 0) != cudaSuccess ||
        cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, copy) != cudaSuccess)
      return RZ_ERR_CUDA;
    return RZ_OK;
  }

  rz_status after_dh(cudaStream_t st, const rz_bf16* dH, int64_t c0, int64_t rows, int32_t d) {
    if (dH_host == nullptr) return RZ_OK;
    const size_t off = static_cast<size_t>(c0) * static_cast<size_t>(d);
    return copy_after(st, dH_host + off, dH + off, static_cast<size_t>(rows) * d * sizeof(rz_bf16));
  }

  rz_status after_dw(cudaStream_t st, const float* dW, int32_t V, int32_t d) {
    if (dW_host == nullptr) return RZ_OK;
    return copy_after(st, dW_host, dW, static_cast<size_t>(V) * d * sizeof(float));
  }

  // Work enqueued on `st` after this waits for every copy enqueued so far.
  rz_status finish(cudaStream_t st) {
    if (cudaEventRecord(ev, copy) != cudaSuccess || cudaStreamWaitEvent(st, ev, 0) != cudaSuccess)
      return RZ_ERR_CUDA;
    return RZ_OK;
  }
};

// Backward of one chunk of rows [c0, c0 + rows), after its forward (e, tile maxima) and
// its kappa: dZ in place, dH rows = dZ W, dW (+)= dZ^T H.  With `out`, the chunk's dH rows
// are copied to host memory right after their contraction.
rz_status run_backward_chunk(const rz_bf16* H, const rz_bf16* W, const int32_t* ids, int64_t c0, int64_t rows,
                             int32_t d, int32_t V, const float* lp, const float* lse, const float* kappa,
                             rz_bf16* dH, float* dW, void* ws, const Layout& L, cudaStream_t stream,
                             Recorder* rec, HostExport* out = nullptr) {
  int* status = at<int>(ws, L.status);
  uint16_t* dz = at<uint16_t>(ws, L.dz);
  const int64_t ldz = padded_vocab(V);

  rec_begin(rec, RZ_KERNEL_DZ, stream);
  {
    dz_from_p_kernel<<<static_cast<unsigned>(rows), kDzThreads, 0, stream>>>(
        lse + c0, lp + c0, kappa + c0, ids + c0, at<float>(ws, L.tile_max), num_vocab_tiles(V), V, ldz, dz);
    if (cudaGetLastError() != cudaSuccess) return RZ_ERR_CUDA;
  }
  rec_end(rec, stream);

  // dH chunk = dZ W: A = dZ (K-major, K = V), B = W (MN-major: d contiguous)
  {
    CUtensorMap mDzK, mWmn;
    if (!make_operand_map(&mDzK, dz, V, rows, static_cast<uint64_t>(ldz) * 2, BM)) return RZ_ERR_CUDA;
    if (!make_operand_map(&mWmn, W, d, V, static_cast<uint64_t>(d) * 2, 64)) return RZ_ERR_CUDA;
    EpiDh e;
    if (!make_store_map(&e.out_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dH + c0 * d, d, rows,
                        static_cast<uint64_t>(d) * 2))
      return RZ_ERR_CUDA;
    e.out_cols = d;
    e.out_rows = rows;
    GemmSched s = make_sched(rows, d, 1, 1, V);
    s.group_n = backward_group_n(s.n_tiles);
    s.l2_pol_a = first_if_few(s.group_n);  // dZ rows, read by the group's tiles of the row block
    const OperandPos pos{0, 0, 0, 0};
    rec_begin(rec, RZ_KERNEL_DH, stream);
    if (launch_gemm<false, true>(mDzK, mWmn, s, pos, e, status, stream) != cudaSuccess) return RZ_ERR_CUDA;
    rec_end(rec, stream);
    if (out != nullptr) {
      const rz_status r = out->after_dh(stream, dH, c0, rows, d);
      if (r != RZ_OK) return r;
    }
  }
  // dW (+)= dZ^T H: A = dZ^T (MN-major: V contiguous), B = H chunk (MN-major: d contiguous)
  {
    CUtensorMap mDzMn, mHmn;
    if (!make_operand_map(&mDzMn, dz, V, rows, static_cast<uint64_t>(ldz) * 2, 64)) return RZ_ERR_CUDA;
    // rows of H past the chunk read as zeros
    if (!make_operand_map(&mHmn, H, d, c0 + rows, static_cast<uint64_t>(d) * 2, 64)) return RZ_ERR_CUDA;
    EpiDw e;
    if (!make_store_map(&e.out_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dW, d, V, static_cast<uint64_t>(d) * 4))
      return RZ_ERR_CUDA;
    e.out_cols = d;
    e.out_rows = V;
    e.accumulate = c0 > 0 ? 1 : 0;
    GemmSched s = make_sched(V, d, 1, 1, rows);
    s.group_n = dw_group_n(s.n_tiles, rows);
    s.l2_pol_a = first_if_few(s.group_n);  // dZ^T
    // the group's columns of the chunk's H
    s.l2_pol_b = keep_if_fits(static_cast<uint64_t>(rows) * std::min<int64_t>(d, s.group_n * BN) * 2);
    const OperandPos pos{0, 0, 0, static_cast<int>(c0)};
    rec_begin(rec, RZ_KERNEL_DW, stream);
    if (launch_gemm<true, true>(mDzMn, mHmn, s, pos, e, status, stream) != cudaSuccess) return RZ_ERR_CUDA;
    rec_end(rec, stream);
  }
  return RZ_OK;
}

}  // namespace
}  // namespace rz

using namespace rz;

extern "C" {
#define RZ_API __attribute__((visibility("default")))

RZ_API const char* rz_status_string(rz_status s) {
  switch (s) {
    case RZ_OK: return "RZ_OK";
    case RZ_ERR_INVALID_ARG: return "RZ_ERR_INVALID_ARG";
    case RZ_ERR_UNSUPPORTED_SHAPE: return "RZ_ERR_UNSUPPORTED_SHAPE";
    case RZ_ERR_WORKSPACE_TOO_SMALL: return "RZ_ERR_WORKSPACE_TOO_SMALL";
    case RZ_ERR_CUDA: return "RZ_ERR_CUDA";
    case RZ_ERR_DEVICE_CHECK: return "RZ_ERR_DEVICE_CHECK";
    case RZ_ERR_DEVICE_TIMEOUT: return "RZ_ERR_DEVICE_TIMEOUT";
  }
  return "RZ_UNKNOWN_STATUS";
}

RZ_API size_t rz_workspace_bytes_logprobs(int64_t n_tok, int32_t d, int32_t V) {
  if (n_tok < 0 || n_tok >= (int64_t{1} << 31) || !shape_ok(d, V)) return 0;
  return make_layout(n_tok, 0, 0, V, Path::Forward).total;
}

RZ_API size_t rz_workspace_bytes_loss(int64_t n_tok, int32_t n_resp, int32_t n_groups, int32_t d, int32_t V) {
  if (n_tok < 1 || n_tok >= (int64_t{1} << 31) || n_resp < 1 || n_groups < 1 || !shape_ok(d, V)) return 0;
  return make_layout(n_tok, n_resp, n_groups, V, Path::Loss).total;
}

RZ_API size_t rz_workspace_bytes_segment_loss(int64_t n_tok, int32_t n_resp, int32_t n_groups) {
  if (n_tok < 1 || n_tok >= (int64_t{1} << 31) || n_resp < 1 || n_groups < 1) return 0;
  return make_layout(n_tok, n_resp, n_groups, 1, Path::LossStage).total;
}

}  // extern "C"

namespace {

// Host checks of the forward entry points (workspace checked by the caller).
rz_status check_forward_args(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids, int64_t n_tok,
                             int32_t d, int32_t V, const float* lp_out, const float* lse_out) {
  if (n_tok < 0 || n_tok >= (int64_t{1} << 31)) return RZ_ERR_INVALID_ARG;
  if (!shape_ok(d, V)) return RZ_ERR_UNSUPPORTED_SHAPE;
  if (n_tok == 0) return RZ_OK;
  if (!H || !W_head || !token_ids || !lp_out) return RZ_ERR_INVALID_ARG;
  if (!aligned(H, 16) || !aligned(W_head, 16) || !aligned(token_ids, 4) || !aligned(lp_out, 4) ||
      (lse_out && !aligned(lse_out, 4)))
    return RZ_ERR_INVALID_ARG;
  return RZ_OK;
}

// The forward on a checked workspace: clear the status word, then the LM head + online
// log-sum-exp and the merge.  inject_timeout (self-test only) enqueues, right after the
// clear, one bounded wait on a barrier nothing arrives on (1 ms limit), which sets the
// timeout bit exactly as a wait inside the forward that gave up would.
rz_status forward_on_workspace(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids, int64_t n_tok,
                               int32_t d, int32_t V, float* lp_out, float* lse_out, void* ws, const Layout& L,
                               cudaStream_t st, bool inject_timeout) {
  if (cudaMemsetAsync(at<int>(ws, L.status), 0, 16, st) != cudaSuccess) return RZ_ERR_CUDA;
  if (inject_timeout) {
    // the status piece is 256 bytes: the waited time goes to byte 16, past the two words
    wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(1000000ull, at<int>(ws, L.status),
                                                   at<unsigned long long>(ws, L.status + 16));
    if (cudaGetLastError() != cudaSuccess) return RZ_ERR_CUDA;
  }
  return run_forward(H, W_head, token_ids, 0, n_tok, d, V, lp_out, lse_out, ws, L, false, st, nullptr, true);
}

}  // namespace

extern "C" {

RZ_API rz_status rz_token_logprobs(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids, int64_t n_tok,
                            int32_t d, int32_t V, float* lp_out, float* lse_out, void* workspace,
                            size_t ws_bytes, void* stream) {
  const rz_status c = check_forward_args(H, W_head, token_ids, n_tok, d, V, lp_out, lse_out);
  if (c != RZ_OK || n_tok == 0) return c;
  if (!workspace || !aligned(workspace, kAlign)) return RZ_ERR_INVALID_ARG;
  const Layout L = make_layout(n_tok, 0, 0, V, Path::Forward);
  if (ws_bytes < L.total) return RZ_ERR_WORKSPACE_TOO_SMALL;
  return forward_on_workspace(H, W_head, token_ids, n_tok, d, V, lp_out, lse_out, workspace, L,
                              static_cast<cudaStream_t>(stream), false);
}

namespace {
rz_status segment_loss_impl(const float* lp, const float* lp_rollout, const float* rewards,
                            const int64_t* seg_offsets, const int32_t* group_ids, int64_t n_tok, int32_t n_resp,
                            int32_t n_groups, const rz_loss_options* options, float* loss, float* kappa_out,
                            float* w_out, void* workspace, size_t ws_bytes, void* stream) {
  if (n_tok < 1 || n_tok >= (int64_t{1} << 31) || n_resp < 1 || n_groups < 1) return RZ_ERR_INVALID_ARG;
  if (!lp || !lp_rollout || !rewards || !seg_offsets || !group_ids || !loss || !kappa_out || !workspace)
    return RZ_ERR_INVALID_ARG;
  if (!aligned(lp, 4) || !aligned(lp_rollout, 4) || !aligned(rewards, 4) || !aligned(seg_offsets, 8) ||
      !aligned(group_ids, 4) || !aligned(loss, 4) || !aligned(kappa_out, 4) || (w_out && !aligned(w_out, 4)) ||
      !aligned(workspace, kAlign))
    return RZ_ERR_INVALID_ARG;
  LossOpts opt;
  if (!resolve_options(options, n_resp, &opt)) return RZ_ERR_INVALID_ARG;
  const Layout L = make_layout(n_tok, n_resp, n_groups, 1, Path::LossStage);
  if (ws_bytes < L.total) return RZ_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(at<int>(workspace, L.status), 0, 16, st) != cudaSuccess) return RZ_ERR_CUDA;
  return run_segment_loss(lp, lp_rollout, rewards, seg_offsets, group_ids, n_tok, n_resp, n_groups, opt, loss,
                          kappa_out, w_out, workspace, L, st, nullptr);
}
}  // namespace

RZ_API rz_status rz_segment_loss(const float* lp, const float* lp_rollout, const float* rewards,
                                 const int64_t* seg_offsets, const int32_t* group_ids, int64_t n_tok, int32_t n_resp,
                                 int32_t n_groups, float* loss, float* kappa_out, float* w_out, void* workspace,
                                 size_t ws_bytes, void* stream) {
  return segment_loss_impl(lp, lp_rollout, rewards, seg_offsets, group_ids, n_tok, n_resp, n_groups, nullptr, loss,
                           kappa_out, w_out, workspace, ws_bytes, stream);
}

RZ_API rz_status rz_segment_loss_ex(const float* lp, const float* lp_rollout, const float* rewards,
                                    const int64_t* seg_offsets, const int32_t* group_ids, int64_t n_tok,
                                    int32_t n_resp, int32_t n_groups, const rz_loss_options* options, float* loss,
                                    float* kappa_out, float* w_out, void* workspace, size_t ws_bytes, void* stream) {
  return segment_loss_impl(lp, lp_rollout, rewards, seg_offsets, group_ids, n_tok, n_resp, n_groups, options, loss,
                           kappa_out, w_out, workspace, ws_bytes, stream);
}

}  // extern "C"

namespace {
// A non-blocking stream per device for host-to-device copies, created on first use.
cudaStream_t copy_stream_for_current_device() {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static cudaStream_t streams[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (streams[dev] == nullptr && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess)
    streams[dev] = nullptr;
  return streams[dev];
}

// Rows of H streamed from host memory: copies of row ranges go out on the copy stream, in
// order, each followed by a record of one event; the compute stream waits on the event
// right after each record is enqueued, so every wait sees the copies enqueued before it.
struct HostRows {
  const rz_bf16* host;
  rz_bf16* dev;
  int64_t d;
  cudaStream_t copy = nullptr;
  cudaEvent_t ev = nullptr;
  int64_t next = 0;  // first row whose copy is not yet enqueued

  HostRows(const rz_bf16* h, rz_bf16* dv, int64_t cols) : host(h), dev(dv), d(cols) {}
  HostRows(const HostRows&) = delete;
  HostRows& operator=(const HostRows&) = delete;
  ~HostRows() {
    if (ev != nullptr) cudaEventDestroy(ev);  // released once its pending records complete
  }

  // The copy stream starts after everything already enqueued on `st` (which may still read
  // the device buffer).
  rz_status start(cudaStream_t st) {
    copy = copy_stream_for_current_device();
    if (copy == nullptr) return RZ_ERR_CUDA;
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) {
      ev = nullptr;
      return RZ_ERR_CUDA;
    }
    if (cudaEventRecord(ev, st) != cudaSuccess || cudaStreamWaitEvent(copy, ev, 0) != cudaSuccess)
      return RZ_ERR_CUDA;
    return RZ_OK;
  }

  // Enqueue the copy of rows [next, upto) and record the event after it.
  rz_status enqueue(int64_t upto) {
    if (upto <= next) return RZ_OK;
    const size_t off = static_cast<size_t>(next) * static_cast<size_t>(d);
    const size_t bytes = static_cast<size_t>(upto - next) * static_cast<size_t>(d) * sizeof(rz_bf16);
    if (cudaMemcpyAsync(dev + off, host + off, bytes, cudaMemcpyHostToDevice, copy) != cudaSuccess ||
        cudaEventRecord(ev, copy) != cudaSuccess)
      return RZ_ERR_CUDA;
    next = upto;
    return RZ_OK;
  }

  // Work enqueued on `st` after this waits for every copy enqueued so far.
  rz_status wait(cudaStream_t st) { return cudaStreamWaitEvent(st, ev, 0) == cudaSuccess ? RZ_OK : RZ_ERR_CUDA; }
};

rz_status loss_fwd_bwd_impl(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids,
                          const float* lp_rollout, const float* rewards, const int64_t* seg_offsets,
                          const int32_t* group_ids, int64_t n_tok, int32_t n_resp, int32_t n_groups, int32_t d,
                          int32_t V, const rz_loss_options* options, float* loss, rz_bf16* dH, float* dW,
                          float* lp_out, float* kappa_out, void* workspace, size_t ws_bytes, void* stream,
                          Recorder* rec, HostRows* host_rows = nullptr, HostExport* host_out = nullptr) {
  if (n_tok < 1 || n_tok >= (int64_t{1} << 31) || n_resp < 1 || n_groups < 1) return RZ_ERR_INVALID_ARG;
  LossOpts opt;
  if (!resolve_options(options, n_resp, &opt)) return RZ_ERR_INVALID_ARG;
  if (!shape_ok(d, V)) return RZ_ERR_UNSUPPORTED_SHAPE;
  if (!H || !W_head || !token_ids || !lp_rollout || !rewards || !seg_offsets || !group_ids || !loss || !dH ||
      !dW || !workspace)
    return RZ_ERR_INVALID_ARG;
  if (!aligned(H, 16) || !aligned(W_head, 16) || !aligned(dH, 16) || !aligned(dW, 16) || !aligned(token_ids, 4) ||
      !aligned(lp_rollout, 4) || !aligned(rewards, 4) || !aligned(seg_offsets, 8) || !aligned(group_ids, 4) ||
      !aligned(loss, 4) || (lp_out && !aligned(lp_out, 4)) || (kappa_out && !aligned(kappa_out, 4)) ||
      !aligned(workspace, kAlign))
    return RZ_ERR_INVALID_ARG;
  const Layout L = make_layout(n_tok, n_resp, n_groups, V, Path::Loss);
  if (ws_bytes < L.total) return RZ_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(at<int>(workspace, L.status), 0, 16, st) != cudaSuccess) return RZ_ERR_CUDA;
  float* lp = lp_out ? lp_out : at<float>(workspace, L.lp);
  float* lse = at<float>(workspace, L.lse);
  float* kappa = kappa_out ? kappa_out : at<float>(workspace, L.kappa);
  rz_status r = run_loss_setup(rewards, seg_offsets, group_ids, n_tok, n_resp, n_groups, opt, workspace, L, st, rec);
  if (r != RZ_OK) return r;
  if (host_out != nullptr) {
    r = host_out->start();
    if (r != RZ_OK) return r;
  }
  if (host_rows != nullptr) {  // the first chunk (every chunk for the gate's first pass)
    r = host_rows->start(st);
    if (r == RZ_OK) r = host_rows->enqueue(opt.gate ? n_tok : std::min<int64_t>(kChunkTokens, n_tok));
    if (r == RZ_OK) r = host_rows->wait(st);
    if (r != RZ_OK) return r;
  }
  if (opt.gate) {
    // the gate needs every token's logprob before any kappa: one forward pass first
    // (same kernels, so the same lp bits as the pass that follows)
    for (int64_t c0 = 0; c0 < n_tok; c0 += kChunkTokens) {
      const int64_t rows = std::min<int64_t>(kChunkTokens, n_tok - c0);
      r = run_forward(H, W_head, token_ids, c0, rows, d, V, lp, lse, workspace, L, false, st, rec);
      if (r != RZ_OK) return r;
    }
    r = run_gate(lp, lp_rollout, seg_offsets, n_resp, opt, workspace, L, st);
    if (r != RZ_OK) return r;
  }
  // chunk by chunk: forward (with the exponentials kept), kappa, backward; the loss
  // partials are per 4096-token block, so the loss does not depend on the chunking
  for (int64_t c0 = 0; c0 < n_tok; c0 += kChunkTokens) {
    const int64_t rows = std::min<int64_t>(kChunkTokens, n_tok - c0);
    if (host_rows != nullptr) {  // the next chunk's copy overlaps this chunk's compute
      r = host_rows->enqueue(std::min<int64_t>(c0 + rows + kChunkTokens, n_tok));
      if (r != RZ_OK) return r;
    }
    r = run_forward(H, W_head, token_ids, c0, rows, d, V, lp, lse, workspace, L, true, st, rec);
    if (r != RZ_OK) return r;
    const int blk0 = static_cast<int>(c0 / kKappaBlockTokens);
    const int nblk = static_cast<int>(ceil_div(rows, kKappaBlockTokens));
    r = run_kappa(lp, lp_rollout, seg_offsets, n_tok, n_resp, blk0, nblk, opt, kappa, nullptr, loss, workspace, L,
                  st, rec);
    if (r != RZ_OK) return r;
    r = run_backward_chunk(H, W_head, token_ids, c0, rows, d, V, lp, lse, kappa, dH, dW, workspace, L, st, rec,
                           host_out);
    if (r != RZ_OK) return r;
    if (host_rows != nullptr && c0 + rows < n_tok) {
      r = host_rows->wait(st);  // before the next chunk's kernels
      if (r != RZ_OK) return r;
    }
  }
  if (host_out == nullptr) return RZ_OK;
  r = host_out->after_dw(st, dW, V, d);
  if (r != RZ_OK) return r;
  return host_out->finish(st);
}

}  // namespace

extern "C" {

RZ_API rz_status rz_loss_fwd_bwd(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids,
                                 const float* lp_rollout, const float* rewards, const int64_t* seg_offsets,
                                 const int32_t* group_ids, int64_t n_tok, int32_t n_resp, int32_t n_groups,
                                 int32_t d, int32_t V, float* loss, rz_bf16* dH, float* dW, float* lp_out,
                                 float* kappa_out, void* workspace, size_t ws_bytes, void* stream) {
  return loss_fwd_bwd_impl(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_tok, n_resp,
                           n_groups, d, V, nullptr, loss, dH, dW, lp_out, kappa_out, workspace, ws_bytes, stream,
                           nullptr);
}

RZ_API rz_status rz_loss_fwd_bwd_ex(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids,
                                    const float* lp_rollout, const float* rewards, const int64_t* seg_offsets,
                                    const int32_t* group_ids, int64_t n_tok, int32_t n_resp, int32_t n_groups,
                                    int32_t d, int32_t V, const rz_loss_options* options, float* loss, rz_bf16* dH,
                                    float* dW, float* lp_out, float* kappa_out, void* workspace, size_t ws_bytes,
                                    void* stream) {
  return loss_fwd_bwd_impl(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_tok, n_resp,
                           n_groups, d, V, options, loss, dH, dW, lp_out, kappa_out, workspace, ws_bytes, stream,
                           nullptr);
}

RZ_API rz_status rz_loss_fwd_bwd_streamed(const rz_bf16* H_host, rz_bf16* H_dev, const rz_bf16* W_head,
                                          const int32_t* token_ids, const float* lp_rollout, const float* rewards,
                                          const int64_t* seg_offsets, const int32_t* group_ids, int64_t n_tok,
                                          int32_t n_resp, int32_t n_groups, int32_t d, int32_t V,
                                          const rz_loss_options* options, float* loss, rz_bf16* dH, float* dW,
                                          float* lp_out, float* kappa_out, void* workspace, size_t ws_bytes,
                                          void* stream) {
  if (H_host == nullptr) return RZ_ERR_INVALID_ARG;
  HostRows rows(H_host, H_dev, d);
  return loss_fwd_bwd_impl(H_dev, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_tok, n_resp,
                           n_groups, d, V, options, loss, dH, dW, lp_out, kappa_out, workspace, ws_bytes, stream,
                           nullptr, &rows);
}

RZ_API rz_status rz_loss_fwd_bwd_host_io(const rz_bf16* H_host, rz_bf16* H_dev, const rz_bf16* W_head,
                                         const int32_t* token_ids, const float* lp_rollout, const float* rewards,
                                         const int64_t* seg_offsets, const int32_t* group_ids, int64_t n_tok,
                                         int32_t n_resp, int32_t n_groups, int32_t d, int32_t V,
                                         const rz_loss_options* options, float* loss, rz_bf16* dH, float* dW,
                                         float* lp_out, float* kappa_out, rz_bf16* dH_host, float* dW_host,
                                         void* workspace, size_t ws_bytes, void* stream) {
  if (H_host == nullptr) return RZ_ERR_INVALID_ARG;
  HostRows rows(H_host, H_dev, d);
  HostExport out(dH_host, dW_host);
  return loss_fwd_bwd_impl(H_dev, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_tok, n_resp,
                           n_groups, d, V, options, loss, dH, dW, lp_out, kappa_out, workspace, ws_bytes, stream,
                           nullptr, &rows, &out);
}

RZ_API int32_t rz_num_launches_loss(int64_t n_tok) {
  if (n_tok < 1) return 0;
  return static_cast<int32_t>(1 + 6 * ceil_div(n_tok, kChunkTokens));
}

RZ_API rz_status rz_loss_fwd_bwd_timed(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids,
                                       const float* lp_rollout, const float* rewards, const int64_t* seg_offsets,
                                       const int32_t* group_ids, int64_t n_tok, int32_t n_resp, int32_t n_groups,
                                       int32_t d, int32_t V, float* loss, rz_bf16* dH, float* dW, float* lp_out,
                                       float* kappa_out, void* workspace, size_t ws_bytes, void* stream,
                                       void* const* launch_events, int32_t* launch_kinds, int32_t capacity,
                                       int32_t* n_launches) {
  if (!launch_events || !launch_kinds || !n_launches || capacity < 0) return RZ_ERR_INVALID_ARG;
  Recorder rec{reinterpret_cast<cudaEvent_t*>(const_cast<void**>(launch_events)), launch_kinds, capacity, 0, false};
  const rz_status r = loss_fwd_bwd_impl(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_tok,
                                        n_resp, n_groups, d, V, nullptr, loss, dH, dW, lp_out, kappa_out, workspace,
                                        ws_bytes, stream, &rec);
  *n_launches = rec.count;
  return r;
}

}  // extern "C"

// ---------------------------------------------------------------- allocation-free variant
//
// Scratch for rz_token_logprobs_noalloc: a fixed device array in this library's module,
// so callers that cannot allocate device memory still get the forward.  Every device
// that loads the library holds these RZ_NOALLOC_SCRATCH_BYTES until the process exits.
// All calls share it, so calls whose GPU work overlaps (other streams, other threads)
// race on it.  The status word at its start is cleared by every call; every other byte a
// call reads has been written earlier in that same call, except after a wait that gave
// up, when the merge writes NaN instead of reading the partials (merge_lse_kernel).
static __device__ __align__(256) uint8_t g_noalloc_scratch[RZ_NOALLOC_SCRATCH_BYTES];

namespace {

// Identifier of the calling thread's current CUDA context (cuCtxGetId: unique for the life
// of the process), or 0 when it cannot be read.  Fetched through the runtime's driver entry
// point query, like the tensor-map encoder, so the library needs no link to libcuda.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device.  Host code only sees a
// host-side stand-in under that name, so the address is looked up with the device
// current (cudaGetSymbolAddress) and cached per device together with the CUDA context it
// belongs to: after the device's context is destroyed and recreated (cudaDeviceReset, or
// a released primary context) the next call sees a new context and looks it up again.
rz_status noalloc_scratch(void** out) {
  static void* addr[kMaxDevices] = {};
  static unsigned long long ctx_of[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RZ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RZ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (addr[dev] == nullptr || ctx == 0 || ctx != ctx_of[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return RZ_ERR_CUDA;
    addr[dev] = p;
    ctx_of[dev] = current_context_id();  // the lookup may have created the context
  }
  *out = addr[dev];
  return RZ_OK;
}

rz_status noalloc_forward(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids, int64_t n_tok,
                          int32_t d, int32_t V, float* lp_out, float* lse_out, void* stream, bool inject_timeout) {
  const rz_status c = check_forward_args(H, W_head, token_ids, n_tok, d, V, lp_out, lse_out);
  if (c != RZ_OK || n_tok == 0) return c;
  const Layout L = make_layout(n_tok, 0, 0, V, Path::Forward);
  if (L.total > static_cast<size_t>(RZ_NOALLOC_SCRATCH_BYTES)) return RZ_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  const rz_status r = noalloc_scratch(&scratch);
  if (r != RZ_OK) return r;
  return forward_on_workspace(H, W_head, token_ids, n_tok, d, V, lp_out, lse_out, scratch, L,
                              static_cast<cudaStream_t>(stream), inject_timeout);
}

}  // namespace

extern "C" {

RZ_API rz_status rz_token_logprobs_noalloc(const rz_bf16* H, const rz_bf16* W_head, const int32_t* token_ids,
                                           int64_t n_tok, int32_t d, int32_t V, float* lp_out, float* lse_out,
                                           void* stream) {
  return noalloc_forward(H, W_head, token_ids, n_tok, d, V, lp_out, lse_out, stream, false);
}

RZ_API rz_status rz_selftest_forward_after_timeout(int32_t use_noalloc_scratch, const rz_bf16* H,
                                                   const rz_bf16* W_head, const int32_t* token_ids, int64_t n_tok,
                                                   int32_t d, int32_t V, float* lp_out, float* lse_out,
                                                   void* workspace, size_t ws_bytes, void* stream) {
  if (use_noalloc_scratch)
    return noalloc_forward(H, W_head, token_ids, n_tok, d, V, lp_out, lse_out, stream, true);
  const rz_status c = check_forward_args(H, W_head, token_ids, n_tok, d, V, lp_out, lse_out);
  if (c != RZ_OK || n_tok == 0) return c;
  if (!workspace || !aligned(workspace, kAlign)) return RZ_ERR_INVALID_ARG;
  const Layout L = make_layout(n_tok, 0, 0, V, Path::Forward);
  if (ws_bytes < L.total) return RZ_ERR_WORKSPACE_TOO_SMALL;
  return forward_on_workspace(H, W_head, token_ids, n_tok, d, V, lp_out, lse_out, workspace, L,
                              static_cast<cudaStream_t>(stream), true);
}

namespace {
int stat_blocks(int64_t n) { return static_cast<int>(ceil_div(n, kStatTokens)); }
// status | StatPartial [blocks] | histogram [2048] | selection state [4] | reduced partial
size_t stats_parts_off() { return kAlign; }
size_t stats_hist_off(int64_t n) { return align_up(stats_parts_off() + sizeof(StatPartial) * stat_blocks(n), kAlign); }
size_t stats_sel_off(int64_t n) { return align_up(stats_hist_off(n) + sizeof(unsigned) * kStatBins, kAlign); }
size_t stats_acc_off(int64_t n) { return align_up(stats_sel_off(n) + 16, kAlign); }
size_t stats_k3_off(int64_t n) { return align_up(stats_acc_off(n) + sizeof(StatPartial), kAlign); }
constexpr int kNormBlocks = 1184;  // 8 per SM on 148 SMs; fixed, so the partial order is fixed
}  // namespace

RZ_API size_t rz_workspace_bytes_ratio_stats(int64_t n_tok, int32_t n_resp) {
  if (n_tok < 1 || n_tok >= (int64_t{1} << 31) || n_resp < 1) return 0;
  return align_up(stats_k3_off(n_tok) + sizeof(double) * 2 * stat_blocks(n_tok), kAlign);
}

RZ_API rz_status rz_ratio_stats(const float* lp, const float* lp_rollout, const int64_t* seg_offsets, int64_t n_tok,
                                int32_t n_resp, const uint8_t* token_mask, double* stats_out,
                                float* resp_mean_ratio_out, void* workspace, size_t ws_bytes, void* stream) {
  if (n_tok < 1 || n_tok >= (int64_t{1} << 31) || n_resp < 1) return RZ_ERR_INVALID_ARG;
  if (!lp || !lp_rollout || !seg_offsets || !stats_out || !workspace) return RZ_ERR_INVALID_ARG;
  if (!aligned(lp, 4) || !aligned(lp_rollout, 4) || !aligned(seg_offsets, 8) || !aligned(stats_out, 8) ||
      (resp_mean_ratio_out && !aligned(resp_mean_ratio_out, 4)) || !aligned(workspace, kAlign))
    return RZ_ERR_INVALID_ARG;
  if (ws_bytes < rz_workspace_bytes_ratio_stats(n_tok, n_resp)) return RZ_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  StatPartial* parts = at<StatPartial>(workspace, stats_parts_off());
  unsigned* hist = at<unsigned>(workspace, stats_hist_off(n_tok));
  unsigned* sel = at<unsigned>(workspace, stats_sel_off(n_tok));
  if (cudaMemsetAsync(workspace, 0, 16, st) != cudaSuccess) return RZ_ERR_CUDA;
  if (cudaMemsetAsync(hist, 0, sizeof(unsigned) * kStatBins, st) != cudaSuccess) return RZ_ERR_CUDA;
  if (cudaMemsetAsync(sel, 0, 16, st) != cudaSuccess) return RZ_ERR_CUDA;
  const int nb = stat_blocks(n_tok);
  StatPartial* acc = at<StatPartial>(workspace, stats_acc_off(n_tok));
  const bool vec = aligned(lp, 16) && aligned(lp_rollout, 16);
  // pass 0 (arithmetic-heavy, few histogram bins) runs one CTA per token block; the radix
  // passes run persistent CTAs, a few per SM, that flush their histograms once
  const int sms = sm_count();
  if (sms <= 0) return RZ_ERR_CUDA;
  const int grid = std::min(nb, kStatCtasPerSm * sms);
  ratio_stats_pass0<<<nb, kStatThreads, 0, st>>>(lp, lp_rollout, token_mask, n_tok, vec, nb, parts, hist);
  ratio_stats_reduce<<<1, 1024, 0, st>>>(parts, nb, acc, sel);
  double* k3_parts = at<double>(workspace, stats_k3_off(n_tok));
  const int nk3 = 2 * nb;  // two k3 half-sums per token block, one from each radix pass
  ratio_stats_select<<<1, kSelectThreads, 0, st>>>(hist, kStatBins, 11, sel, acc, 0, stats_out, k3_parts, nk3);
  ratio_stats_pass<0><<<grid, kStatThreads, 0, st>>>(lp, lp_rollout, token_mask, n_tok, vec, nb, sel, 21, 10, 0x7ffu,
                                                     hist, k3_parts);
  ratio_stats_select<<<1, kSelectThreads, 0, st>>>(hist, kStatBins, 11, sel, acc, 0, stats_out, k3_parts, nk3);
  ratio_stats_pass<1><<<grid, kStatThreads, 0, st>>>(lp, lp_rollout, token_mask, n_tok, vec, nb, sel, 10, 0, 0x3ffu,
                                                     hist, k3_parts);
  ratio_stats_select<<<1, kSelectThreads, 0, st>>>(hist, 1024, 10, sel, acc, 1, stats_out, k3_parts, nk3);
  if (resp_mean_ratio_out != nullptr)
    response_mean_ratio_kernel<<<static_cast<unsigned>(ceil_div(n_resp, 8)), 256, 0, st>>>(
        lp, lp_rollout, token_mask, seg_offsets, n_resp, resp_mean_ratio_out);
  return cudaGetLastError() == cudaSuccess ? RZ_OK : RZ_ERR_CUDA;
}

RZ_API size_t rz_workspace_bytes_grad_norms(void) { return align_up(sizeof(double) * 2 * kNormBlocks, kAlign); }

RZ_API rz_status rz_grad_norms(const rz_bf16* dH, const float* dW, int64_t n_tok, int32_t d, int32_t V,
                               double* norms_out, void* workspace, size_t ws_bytes, void* stream) {
  if (n_tok < 0 || d < 1 || V < 0 || !norms_out || !workspace) return RZ_ERR_INVALID_ARG;
  if ((n_tok > 0 && !dH) || (V > 0 && !dW) || !aligned(norms_out, 8) || !aligned(workspace, kAlign))
    return RZ_ERR_INVALID_ARG;
  if (ws_bytes < rz_workspace_bytes_grad_norms()) return RZ_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  double* partials = static_cast<double*>(workspace);
  sumsq_kernel<<<kNormBlocks, 256, 0, st>>>(dH, n_tok * d, 1, partials);
  sumsq_kernel<<<kNormBlocks, 256, 0, st>>>(dW, static_cast<int64_t>(V) * d, 0, partials + kNormBlocks);
  sqrt_sum_kernel<<<1, 32, 0, st>>>(partials, kNormBlocks, norms_out);
  sqrt_sum_kernel<<<1, 32, 0, st>>>(partials + kNormBlocks, kNormBlocks, norms_out + 1);
  return cudaGetLastError() == cudaSuccess ? RZ_OK : RZ_ERR_CUDA;
}

RZ_API rz_status rz_quantize_rows_e4m3(const rz_bf16* X, int64_t rows, int32_t d, uint8_t* X8, float* scale,
                                       void* stream) {
  if (rows < 0 || rows >= (int64_t{1} << 31) || d < 1) return RZ_ERR_INVALID_ARG;
  if (rows == 0) return RZ_OK;
  if (!X || !X8 || !scale || !aligned(X, 2) || !aligned(scale, 4)) return RZ_ERR_INVALID_ARG;
  quantize_rows_e4m3_kernel<<<static_cast<unsigned>(rows), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(X), d, X8, scale);
  return cudaGetLastError() == cudaSuccess ? RZ_OK : RZ_ERR_CUDA;
}

RZ_API rz_status rz_token_logprobs_fp8(const uint8_t* H8, const float* h_scale, const uint8_t* W8,
                                       const float* w_scale, const int32_t* token_ids, int64_t n_tok, int32_t d,
                                       int32_t V, float* lp_out, float* lse_out, void* workspace, size_t ws_bytes,
                                       void* stream) {
  if (n_tok < 0 || n_tok >= (int64_t{1} << 31)) return RZ_ERR_INVALID_ARG;
  if (!shape_ok(d, V) || d % BK_FP8 != 0) return RZ_ERR_UNSUPPORTED_SHAPE;
  if (n_tok == 0) return RZ_OK;
  if (!H8 || !h_scale || !W8 || !w_scale || !token_ids || !lp_out || !workspace) return RZ_ERR_INVALID_ARG;
  if (!aligned(H8, 16) || !aligned(W8, 16) || !aligned(h_scale, 4) || !aligned(w_scale, 4) ||
      !aligned(token_ids, 4) || !aligned(lp_out, 4) || (lse_out && !aligned(lse_out, 4)) ||
      !aligned(workspace, kAlign))
    return RZ_ERR_INVALID_ARG;
  const Layout L = make_layout(n_tok, 0, 0, V, Path::Forward);
  if (ws_bytes < L.total) return RZ_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(at<int>(workspace, L.status), 0, 16, st) != cudaSuccess) return RZ_ERR_CUDA;
  return run_forward_fp8(H8, h_scale, W8, w_scale, token_ids, n_tok, d, V, lp_out, lse_out, workspace, L, st);
}

RZ_API size_t rz_mxfp4_scale_bytes(int64_t rows, int32_t d) {
  if (rows < 0 || rows >= (int64_t{1} << 31) || d < 256 || d > 32768 || d % 256 != 0) return 0;
  return static_cast<size_t>(mxfp4_scale_bytes(rows, d));
}

RZ_API rz_status rz_quantize_rows_mxfp4(const rz_bf16* X, int64_t rows, int32_t d, uint8_t* X4, uint8_t* scales,
                                        void* stream) {
  if (rows < 0 || rows >= (int64_t{1} << 31)) return RZ_ERR_INVALID_ARG;
  if (d < 256 || d > 32768 || d % 256 != 0) return RZ_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return RZ_OK;
  if (!X || !X4 || !scales || !aligned(X, 16) || !aligned(X4, 16)) return RZ_ERR_INVALID_ARG;
  const int64_t padded = (rows + 255) / 256 * 256;
  const int64_t threads = padded * (d / kMxBlock);
  quantize_rows_mxfp4_kernel<<<static_cast<unsigned>(ceil_div(threads, 256)), 256, 0,
                               static_cast<cudaStream_t>(stream)>>>(reinterpret_cast<const __nv_bfloat16*>(X), rows,
                                                                    d, padded, X4, scales);
  return cudaGetLastError() == cudaSuccess ? RZ_OK : RZ_ERR_CUDA;
}

RZ_API rz_status rz_token_logprobs_mxfp4(const uint8_t* H4, const uint8_t* h_scales, const uint8_t* W4,
                                         const uint8_t* w_scales, const int32_t* token_ids, int64_t n_tok, int32_t d,
                                         int32_t V, float* lp_out, float* lse_out, void* workspace, size_t ws_bytes,
                                         void* stream) {
  if (n_tok < 0 || n_tok >= (int64_t{1} << 31)) return RZ_ERR_INVALID_ARG;
  if (!shape_ok(d, V) || d < 256 || d % 256 != 0) return RZ_ERR_UNSUPPORTED_SHAPE;
  if (n_tok == 0) return RZ_OK;
  if (!H4 || !h_scales || !W4 || !w_scales || !token_ids || !lp_out || !workspace) return RZ_ERR_INVALID_ARG;
  if (!aligned(H4, 16) || !aligned(W4, 16) || !aligned(h_scales, 16) || !aligned(w_scales, 16) ||
      !aligned(token_ids, 4) || !aligned(lp_out, 4) || (lse_out && !aligned(lse_out, 4)) ||
      !aligned(workspace, kAlign))
    return RZ_ERR_INVALID_ARG;
  const Layout L = make_layout(n_tok, 0, 0, V, Path::Forward);
  if (ws_bytes < L.total) return RZ_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(at<int>(workspace, L.status), 0, 16, st) != cudaSuccess) return RZ_ERR_CUDA;
  return run_forward_mxfp4(H4, h_scales, W4, w_scales, token_ids, n_tok, d, V, lp_out, lse_out, workspace, L, st);
}

RZ_API rz_status rz_sum_shards_f32(const float* stacked, int32_t nshards, int64_t count, float* out, void* stream) {
  if (nshards < 1 || count < 0 || count > (int64_t{1} << 40)) return RZ_ERR_INVALID_ARG;
  if (count == 0) return RZ_OK;
  if (!stacked || !out || !aligned(stacked, 4) || !aligned(out, 4)) return RZ_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return RZ_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ceil_div(count, 256), int64_t{8} * sms));
  sum_shards_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(stacked, nshards, count, out);
  return cudaGetLastError() == cudaSuccess ? RZ_OK : RZ_ERR_CUDA;
}

RZ_API rz_status rz_selftest_wait_timeout(uint64_t limit_ns, void* workspace, size_t ws_bytes,
                                          uint64_t* waited_ns_out, void* stream) {
  if (!workspace || ws_bytes < 256 || !aligned(workspace, kAlign) || limit_ns > 10000000000ull)
    return RZ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, 16, st) != cudaSuccess) return RZ_ERR_CUDA;
  unsigned long long* waited = at<unsigned long long>(workspace, 16);
  wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(limit_ns, static_cast<int*>(workspace), waited);
  if (cudaGetLastError() != cudaSuccess) return RZ_ERR_CUDA;
  if (waited_ns_out != nullptr) {
    unsigned long long w = 0;
    if (cudaMemcpyAsync(&w, waited, sizeof(w), cudaMemcpyDeviceToHost, st) != cudaSuccess) return RZ_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return RZ_ERR_CUDA;
    *waited_ns_out = w;
  }
  return RZ_OK;
}

RZ_API rz_status rz_read_device_status(const void* workspace, void* stream, int32_t* bits_out) {
  if (!workspace) return RZ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return RZ_ERR_CUDA;
  int32_t bits = 0;
  if (cudaMemcpy(&bits, workspace, sizeof(bits), cudaMemcpyDeviceToHost) != cudaSuccess) return RZ_ERR_CUDA;
  if (bits_out) *bits_out = bits;
  if (bits & RZ_DEV_WAIT_TIMEOUT) return RZ_ERR_DEVICE_TIMEOUT;
  if (bits) return RZ_ERR_DEVICE_CHECK;
  return RZ_OK;
}

}  // extern "C"
