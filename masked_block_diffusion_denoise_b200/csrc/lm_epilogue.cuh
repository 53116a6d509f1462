// Fused vocabulary reduction of the LM head (non-materialised scoring, the
// "chunked" head scoring of the Nemotron guide, section 5.3): each GEMM tile
// of logits is reduced, per row, to
//   m  = max z, s = sum e^(z-m), t = sum e^(z-m) (z-m)
//   (g, idx, zw): the winning column -- the argmax of z (greedy, lowest index
//   on ties) or of z + Gumbel noise (sampling) -- and its scaled logit,
// with z = logit / T (T = 1 for greedy) and the mask id excluded.  Partials of
// all tiles of a row are combined afterwards; confidence = e^(zw - M) / S and
// entropy H = log S - T/S (nats).
#pragma once

#include <math_constants.h>

#include "common.cuh"

namespace dlm {

struct LmPart {
  float m, s, t, g, zw;
  int idx;
};

// Partials are stored field-major within a row, [row][kLmFields][n_part]
// floats (idx as its int bits): a warp that reads one field of 32
// consecutive partials of a row reads one contiguous 128-byte line.
constexpr int kLmFields = 6;

enum { LM_GREEDY = 0, LM_SAMPLE_FIXED = 1, LM_SAMPLE_ANNEAL = 2 };

struct LmEpi {
  int V;          // vocabulary (columns >= V are excluded)
  int mask_id;    // excluded column, < 0 for none
  int C;          // canvas length: row r is position r % C of canvas r / C
  int S;          // step budget (anneal)
  int mode;       // LM_GREEDY / LM_SAMPLE_FIXED / LM_SAMPLE_ANNEAL
  float inv_temp; // LM_SAMPLE_FIXED
  float t_max, t_min;
  uint32_t seed_lo, seed_hi;
  const int32_t* step;   // [B] steps taken (sampling counter and anneal)
  int n_tiles;    // partials per row
  // e4m3 LM head: logit = acc * (row_scale[r] * col_scale[v]); null otherwise
  const float* row_scale;
  const float* col_scale;   // padded with zeros to whole vocabulary tiles
};

struct RowState {
  float m, s, t, g, zw;
  int idx;
};

__device__ __forceinline__ void rs_init(RowState& r) {
  r.m = -CUDART_INF_F;
  r.s = 0.f;
  r.t = 0.f;
  r.g = -CUDART_INF_F;
  r.zw = -CUDART_INF_F;
  r.idx = 0x7fffffff;
}

// 1/T of a row, float32 with explicit rounding so that the host can repeat it
__device__ __forceinline__ float lm_inv_temp(const LmEpi& e, int step) {
  if (e.mode == LM_SAMPLE_FIXED) return e.inv_temp;
  if (e.mode == LM_SAMPLE_ANNEAL) {
    float T = e.t_max;
    if (e.S > 1) {
      const float frac = __fdiv_rn((float)step, (float)(e.S - 1));
      T = __fadd_rn(e.t_max, __fmul_rn(__fsub_rn(e.t_min, e.t_max), frac));
    }
    return __frcp_rn(T);
  }
  return 1.f;
}

// three-input maximum (sm_100 max.f32 with three operands)
__device__ __forceinline__ float lm_max3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

// Greedy fold of a chunk with no excluded column (the common case: every
// chunk but the one holding the mask id and the vocabulary's ragged end).
// The same state as the general path below, with less work per logit, which
// matters on a power-capped GPU where the epilogue's instructions take power
// from the tensor cores: the chunk maximum by three-input maxima; the
// argmax searched only when the chunk beats the row's best (first
// occurrence, as the general path); then per logit one FFMA (x = z log2 e -
// m log2 e), one exponential, one add for s and one FFMA for the entropy
// term, summed in base 2 and scaled by ln 2 once per chunk.
template <int N>
__device__ __forceinline__ void rs_update_greedy_clean(RowState& r, const float (&v)[N],
                                                       int col0) {
  static_assert(N % 4 == 0, "chunks of 4k logits");
  float mx[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
  for (int j = 4; j + 8 <= N; j += 8)
#pragma unroll
    for (int k = 0; k < 4; ++k) mx[k] = lm_max3(mx[k], v[j + k], v[j + 4 + k]);
  if constexpr (N % 8 == 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) mx[k] = fmaxf(mx[k], v[N - 4 + k]);
  }
  const float cmax = fmaxf(lm_max3(mx[0], mx[1], mx[2]), mx[3]);
  if (!(cmax > -CUDART_INF_F)) return;   // no finite logit (as the general path)
  if (cmax > r.g) {   // columns arrive in increasing order: on equal values the earlier wins
    int carg = 0;
#pragma unroll
    for (int j = N - 1; j >= 0; --j) carg = v[j] == cmax ? j : carg;
    r.g = cmax;
    r.zw = cmax;
    r.idx = col0 + carg;
  }
  if (cmax > r.m) {
    if (r.m != -CUDART_INF_F) {
      const float a = __expf(r.m - cmax);
      r.t = (r.t + r.s * (r.m - cmax)) * a;
      r.s *= a;
    }
    r.m = cmax;
  }
  constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
  const float m2 = r.m * kLog2e;
  float s4[4] = {0.f, 0.f, 0.f, 0.f}, t4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float x = fmaf(v[j], kLog2e, -m2);   // (z - m) log2 e
    const float ex = fast_exp2(x);
    s4[j & 3] += ex;
    t4[j & 3] = fmaf(ex, x, t4[j & 3]);
  }
  r.s += (s4[0] + s4[1]) + (s4[2] + s4[3]);
  r.t = fmaf((t4[0] + t4[1]) + (t4[2] + t4[3]), kLn2, r.t);
}

// Fold N consecutive logits (columns col0 .. col0+N-1, col0 % 4 == 0) of one
// row into the row state.  canvas / pos / step locate the row for the
// sampling counter.
template <int N>
__device__ __forceinline__ void rs_update(RowState& r, const float (&v)[N], int col0,
                                          float inv_t, const LmEpi& e, int canvas, int pos,
                                          int step) {
  if (e.mode == LM_GREEDY && col0 + N <= e.V && (unsigned)(e.mask_id - col0) >= (unsigned)N) {
    rs_update_greedy_clean<N>(r, v, col0);
    return;
  }
  float z[N];
  float cmax = -CUDART_INF_F;
  int carg = 0;
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const int col = col0 + j;
    float zj = (e.mode == LM_GREEDY) ? v[j] : __fmul_rn(v[j], inv_t);
    if (col >= e.V || col == e.mask_id) zj = -CUDART_INF_F;
    z[j] = zj;
    if (zj > cmax) {
      cmax = zj;
      carg = j;
    }
  }
  if (cmax == -CUDART_INF_F) return;
  if (cmax > r.m) {
    if (r.m != -CUDART_INF_F) {
      const float a = __expf(r.m - cmax);
      r.t = (r.t + r.s * (r.m - cmax)) * a;
      r.s *= a;
    }
    r.m = cmax;
  }
  // branch-free: masked columns contribute exactly zero (selects, not branches,
  // so independent work of the chunk can interleave)
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const bool valid = z[j] != -CUDART_INF_F;
    const float d = valid ? z[j] - r.m : 0.f;
    const float ex = valid ? __expf(d) : 0.f;
    r.s += ex;
    r.t = fmaf(ex, d, r.t);
  }
  if (e.mode == LM_GREEDY) {
    // columns arrive in increasing order: on equal values the earlier wins
    const bool better = cmax > r.g;
    r.g = better ? cmax : r.g;
    r.zw = better ? cmax : r.zw;
    r.idx = better ? col0 + carg : r.idx;
  } else {
    U32x4 w[N / 4];
#pragma unroll
    for (int j4 = 0; j4 < N / 4; ++j4)
      w[j4] = philox10(U32x4{(uint32_t)canvas, (uint32_t)step, (uint32_t)pos,
                             (uint32_t)((col0 >> 2) + j4)},
                       e.seed_lo, e.seed_hi);
#pragma unroll
    for (int j4 = 0; j4 < N / 4; ++j4) {
      const uint32_t ws[4] = {w[j4].a, w[j4].b, w[j4].c, w[j4].d};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float zj = z[4 * j4 + q];
        const float gj = zj + gumbel_from_bits(ws[q]);   // -inf stays -inf
        const bool better = gj > r.g;                     // ties keep the lower index
        r.g = better ? gj : r.g;
        r.zw = better ? zj : r.zw;
        r.idx = better ? col0 + 4 * j4 + q : r.idx;
      }
    }
  }
}

// partial j of row `row` (n_part partials per row)
__device__ __forceinline__ void rs_store(float* part, int n_part, size_t row, int j,
                                         const RowState& r) {
  float* d = part + row * kLmFields * (size_t)n_part + j;
  d[0] = r.m;
  d[n_part] = r.s;
  d[2 * n_part] = r.t;
  d[3 * n_part] = r.g;
  d[4 * n_part] = r.zw;
  d[5 * n_part] = __int_as_float(r.idx);
}

// combine two partial states (the order of arguments fixes the tie rule:
// equal winners keep the lower index)
__device__ __forceinline__ RowState rs_combine(const RowState& a, const RowState& b) {
  RowState c;
  const float M = fmaxf(a.m, b.m);
  if (M == -CUDART_INF_F) {
    rs_init(c);
    return c;
  }
  float s = 0.f, t = 0.f;
  if (a.m != -CUDART_INF_F) {
    const float w = __expf(a.m - M);
    s += a.s * w;
    t += (a.t + a.s * (a.m - M)) * w;
  }
  if (b.m != -CUDART_INF_F) {
    const float w = __expf(b.m - M);
    s += b.s * w;
    t += (b.t + b.s * (b.m - M)) * w;
  }
  c.m = M;
  c.s = s;
  c.t = t;
  const bool take_b = (b.g > a.g) || (b.g == a.g && b.idx < a.idx);
  c.g = take_b ? b.g : a.g;
  c.zw = take_b ? b.zw : a.zw;
  c.idx = take_b ? b.idx : a.idx;
  return c;
}

}  // namespace dlm
