// rz_epilogues.cuh -- the epilogues that turn the tensor-core engine into the three
// contractions of the path:
//
//   EpiLse<false>  fused LM head + online log-sum-exp + gather (logits stay on chip);
//                  EpiLse<false, true> the same with split partial sums (the fp8 forward)
//   EpiLse<true>   the same, also keeping exp(z - tile max) (fp16) for the backward
//   EpiDh          dH = dZ W tile, TMA-stored as bf16
//   EpiDw          dW (+)= dZ^T H tile, TMA-stored / TMA-reduce-added in chunk order
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

// Fold one tile's (maximum, sum of exponentials) pair into a row's running pair, in a fixed
// rounding order (explicit fp32 operations, no contraction left to the compiler), so that the
// epilogue and a later merge that replays the same folds give the same bits:
//   m' = max(m, tmax);  s' = s 2^((m - m') log2 e) + tsum 2^((tmax - m') log2 e)
// From (m, s) = (-inf, 0) the first fold gives exactly (tmax, tsum).
__device__ __forceinline__ void lse_fold(float& m, float& s, float tmax, float tsum) {
  const float m_new = fmaxf(m, tmax);
  s = __fmaf_rn(s, ex2_approx(__fmul_rn(m - m_new, kLog2e)), __fmul_rn(tsum, ex2_approx(__fmul_rn(tmax - m_new, kLog2e))));
  m = m_new;
}

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
template <bool STORE_P, bool SPLIT = false>
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
  const float* row_scale;  // nullable: logit = row_scale[row] * (acc * col_scale[col]) (scaled fp8 operands)
  const float* col_scale;
  int col_scale_vec;       // col_scale is 16-byte aligned: read it four columns at a time

  struct State {
    float m, s, rs;
    int y;
    int64_t row;
    float4 cs_next[2];  // scaled operands: this lane's 8 column scales of tile cs_next_tile
    int cs_next_tile;
  };

  __device__ __forceinline__ void begin_unit(State& st, int mb, int, int r) const {
    st.row = static_cast<int64_t>(mb) * BM + r;
    st.y = st.row < rows ? __ldg(ids + st.row) : -1;
    st.m = -INFINITY;
    st.s = 0.0f;
    st.rs = (row_scale != nullptr && st.row < rows) ? __ldg(row_scale + st.row) : 1.0f;
    st.cs_next_tile = -1;
  }

  // Lane l's share of tile nt's 256 column scales: columns nt*256 + 8l .. 8l+7 (0 past V).
  __device__ __forceinline__ void fetch_col_scales(int nt, int lane, float4 (&cs)[2]) const {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = nt * BN + 8 * lane + 4 * h;
      if (col_scale_vec && c + 3 < V) {
        cs[h] = __ldg(reinterpret_cast<const float4*>(col_scale + c));
      } else {
        cs[h].x = c < V ? __ldg(col_scale + c) : 0.0f;
        cs[h].y = c + 1 < V ? __ldg(col_scale + c + 1) : 0.0f;
        cs[h].z = c + 2 < V ? __ldg(col_scale + c + 2) : 0.0f;
        cs[h].w = c + 3 < V ? __ldg(col_scale + c + 3) : 0.0f;
      }
    }
  }

  // Scaled operands: put tile nt's column scales into the warp's shared buffer (from the
  // registers filled one tile ahead, else straight from memory) and start fetching tile
  // nt + 1's, so the global-memory latency of the scales is hidden behind a tile of work.
  __device__ __forceinline__ void stage_col_scales(State& st, int nt, int lane, float* buf) const {
    float4 cur[2];
    if (st.cs_next_tile == nt) {
      cur[0] = st.cs_next[0];
      cur[1] = st.cs_next[1];
    } else {
      fetch_col_scales(nt, lane, cur);
    }
    __syncwarp();  // every lane is done with the previous tile's scales
    reinterpret_cast<float4*>(buf)[2 * lane] = cur[0];
    reinterpret_cast<float4*>(buf)[2 * lane + 1] = cur[1];
    __syncwarp();
    if (nt + 1 < n_tiles) {
      fetch_col_scales(nt + 1, lane, st.cs_next);
      st.cs_next_tile = nt + 1;
    }
  }

  // Scaled operands: y = acc * col_scale (one rounding), the scales of the chunk's 32
  // columns read from the warp's shared buffer (broadcast); the positive row scale is kept
  // out of the per-logit work (see tile).
  __device__ __forceinline__ void scale_columns(const float* buf, int c, float (&v)[32]) const {
    if (col_scale == nullptr) return;  // uniform
    const float4* cs4 = reinterpret_cast<const float4*>(buf + c * 32);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 cs = cs4[q];
      v[4 * q] *= cs.x;
      v[4 * q + 1] *= cs.y;
      v[4 * q + 2] *= cs.z;
      v[4 * q + 3] *= cs.w;
    }
  }

  __device__ __forceinline__ void tile(State& st, uint32_t taddr, int mb, int nt, int r, int lane,
                                       WarpStage& stage) const {
    // chunks of 32 columns holding at least one column < V (uniform across the warp)
    const int nch = min(BN / 32, (V - nt * BN + 31) / 32);
    // The logits are z = rs * y with y = acc (bf16) or acc * col_scale (fp8) and rs the row
    // scale (1 for bf16).  rs > 0, so max z = rs * max y exactly, and
    // exp(z - max z) = 2^((y - max y) * (rs log2 e)); with rs = 1 this is the plain form.
    const float c2 = st.rs * kLog2e;
    // scaled operands only (never with STORE_P, whose staging slots the buffer shares)
    float* cs_buf = reinterpret_cast<float*>(stage.base);
    if (!STORE_P && col_scale != nullptr) stage_col_scales(st, nt, lane, cs_buf);
    // pass 1: tile maximum of y over the valid columns.  SPLIT (the fp8 forward, whose MMAs
    // take half the time of bf16's, so its epilogue is relatively twice as heavy): four
    // partial maxima, column j into partial j % 4 (a maximum does not depend on the order),
    // and no per-column test on chunks wholly inside V.
    float ymax = -INFINITY;
    float ym[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    tmem_for_chunks(taddr, nch, [&](int c, float (&v)[32]) {
      const int col0 = nt * BN + c * 32;
      scale_columns(cs_buf, c, v);
      if constexpr (SPLIT) {
        if (col0 + 32 <= V) {
#pragma unroll
          for (int j = 0; j < 32; ++j) ym[j & 3] = fmaxf(ym[j & 3], v[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < V) ym[j & 3] = fmaxf(ym[j & 3], v[j]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < V) ymax = fmaxf(ymax, v[j]);
      }
    });
    if constexpr (SPLIT) ymax = fmaxf(fmaxf(ym[0], ym[1]), fmaxf(ym[2], ym[3]));
    // pass 2: exponentials relative to the tile maximum, their sum, the gather.  The sum runs
    // in column order; SPLIT: as four partial sums (column j into partial j % 4) added
    // pairwise at the end, a fixed order per row with a quarter of the dependent adds.
    float tsum = 0.0f;
    float ts[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    tmem_for_chunks(taddr, nch, [&](int c, float (&v)[32]) {
      const int col0 = nt * BN + c * 32;
      scale_columns(cs_buf, c, v);
      const unsigned off = static_cast<unsigned>(st.y - col0);
      if (off < 32u) {
        float z = v[0];
#pragma unroll
        for (int j = 1; j < 32; ++j) z = (static_cast<unsigned>(j) == off) ? v[j] : z;
        zy[st.row] = st.rs * z;
      }
      float e[32];
      if constexpr (SPLIT) {
        if (col0 + 32 <= V) {
#pragma unroll
          for (int j = 0; j < 32; ++j) e[j] = ex2_approx((v[j] - ymax) * c2);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) e[j] = (col0 + j < V) ? ex2_approx((v[j] - ymax) * c2) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) ts[j & 3] += e[j];
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          e[j] = (col0 + j < V) ? ex2_approx((v[j] - ymax) * c2) : 0.0f;
          tsum += e[j];
        }
      }
      if constexpr (STORE_P) {
        uint4 row[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          row[q] = make_uint4(pack_half2(e[8 * q], e[8 * q + 1]), pack_half2(e[8 * q + 2], e[8 * q + 3]),
                              pack_half2(e[8 * q + 4], e[8 * q + 5]), pack_half2(e[8 * q + 6], e[8 * q + 7]));
        stage.store_rows(&p_map, lane, row, col0, mb * BM + (r - lane), rows);
      }
    });
    if constexpr (SPLIT) tsum = (ts[0] + ts[1]) + (ts[2] + ts[3]);
    const float tmax = st.rs * ymax;
    lse_fold(st.m, st.s, tmax, tsum);
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

// dH tile: fp32 accumulator -> bf16, TMA-stored into a [rows, d] map of the chunk.
struct EpiDh {
  CUtensorMap out_map;  // bf16 [rows, d], box 32 x 32, 64-byte swizzle

  struct State {};

  __device__ __forceinline__ void begin_unit(State&, int, int, int) const {}

  __device__ __forceinline__ void tile(State&, uint32_t taddr, int mb, int nt, int r, int lane,
                                       WarpStage& stage) const {
    const int nch = min(BN / 32, (out_cols - nt * BN) / 32);
    tmem_for_chunks(taddr, nch, [&](int c, float (&v)[32]) {
      const int col0 = nt * BN + c * 32;
      uint4 row[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        row[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                            pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
      stage.store_rows(&out_map, lane, row, col0, mb * BM + (r - lane), out_rows);
    });
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
    const int nch = min(BN / 32, (out_cols - nt * BN) / 32);
    tmem_for_chunks(taddr, nch, [&](int c, float (&v)[32]) {
      const int col0 = nt * BN + c * 32;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint4 row[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          row[q] = make_uint4(__float_as_uint(v[16 * h + 4 * q]), __float_as_uint(v[16 * h + 4 * q + 1]),
                              __float_as_uint(v[16 * h + 4 * q + 2]), __float_as_uint(v[16 * h + 4 * q + 3]));
        stage.store_rows(&out_map, lane, row, col0 + 16 * h, mb * BM + (r - lane), out_rows, accumulate != 0);
      }
    });
  }

  __device__ __forceinline__ void end_unit(const State&, int, int, int) const {}
};

}  // namespace rz
