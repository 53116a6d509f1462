// Canvas attention: every canvas position of sequence b attends, with one
// joint softmax and no mask, to the cached prefix of b and all canvas
// positions (Nemotron guide, section 6: bidirectional mask over the block;
// course "Diffusion LLMs", section 14: the block reads the finished prefix
// and all of its own positions).  Canvas K/V are written by the projection
// epilogue into cache slots len..len+C-1, so the keys of sequence b are cache
// slots [0, len_b + C).
//
// bf16 kernel: one CTA per (key split, 128-query-row tile, sequence x KV
// head).  The query rows of a CTA are the G = H/Hkv query heads that share
// the KV head times the C canvas positions (GQA grouping), so each K/V tile
// is read once for all of them.  A producer warp streams 64-key K and V
// tiles from HBM with TMA (128-byte swizzle) through a 4-stage ring; eight
// consumer warps own 16 query rows each and run QK^T and PV with
// mma.sync m16n8k16 (fp32 accumulate), keeping the online-softmax state
// (running max, sum) in registers with quad shuffles.  Splits write
// unnormalised partials that a second kernel combines (log-sum-exp).
#include <math_constants.h>

#include "kernels.h"

namespace dlm {
namespace {

constexpr int kDh = 128;
constexpr int kKT = 64;          // keys per tile
constexpr int kStages = 4;
constexpr int kWarps = 8;        // consumer warps
constexpr int kRowsCta = 16 * kWarps;
constexpr int kQBytes = kRowsCta * kDh * 2;       // 32 KB
constexpr int kTileBytes = kKT * kDh * 2;         // 16 KB (K or V)
constexpr int kStageBytes = 2 * kTileBytes;       // K + V
constexpr int kAttnSmem = kQBytes + kStages * kStageBytes + 1024 + 128;

struct AttnParams {
  const __nv_bfloat16* q;
  __nv_bfloat16* o;
  float* opart;
  float2* ml;
  const int32_t* lens;
  const uint8_t* done;
  const int* n_active;
  int* err;
  int H, Hkv, G, C, R, chunk, nsplit;
  float scale_log2;
};

__global__ void __launch_bounds__(32 * (kWarps + 1), 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const AttnParams p) {
  pdl_wait_then_release();
  if (p.n_active != nullptr && *p.n_active == 0) return;
  const int split = blockIdx.x, rt = blockIdx.y, bg = blockIdx.z;
  const int b = bg / p.Hkv, g = bg - b * p.Hkv;
  if (p.done != nullptr && p.done[b]) return;
  const int n_keys = p.lens[b] + p.C;
  const int k_begin = split * p.chunk;
  if (k_begin >= n_keys) return;
  const int k_end = min(k_begin + p.chunk, n_keys);
  const int n_tiles = (k_end - k_begin + kKT - 1) / kKT;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qs = smem;
  uint8_t* ring = smem + kQBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // query tile -> shared memory, two 64-column halves, 128-byte swizzle
  for (int idx = tid; idx < kRowsCta * 16; idx += blockDim.x) {
    const int lr = idx >> 4, ch = idx & 15;
    const int r = rt * kRowsCta + lr;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < p.R) {
      const int i = r / p.G, hh = r - i * p.G;
      const __nv_bfloat16* src =
          p.q + ((size_t)(b * p.C + i) * p.H + (g * p.G + hh)) * kDh + ch * 8;
      val = *reinterpret_cast<const uint4*>(src);
    }
    *reinterpret_cast<uint4*>(qs + (ch >> 3) * (kRowsCta * 128) + sw128_off(lr, ch & 7)) = val;
  }
  __syncthreads();

  const int plane = b * p.Hkv + g;
  if (warp == kWarps) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
      int issued = 0;
      bool ok = true;
      for (int t = 0; t < n_tiles; ++t) {
        const int stage = t % kStages;
        const uint32_t phase = (uint32_t)((t / kStages) & 1);
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* ks = ring + stage * kStageBytes;
        uint8_t* vs = ks + kTileBytes;
        const int key0 = k_begin + t * kKT;
        mbar_arrive_expect_tx(&full[stage], kStageBytes);
        tma_load_3d(ks, &tmK, &full[stage], 0, key0, plane);
        tma_load_3d(ks + kTileBytes / 2, &tmK, &full[stage], 64, key0, plane);
        tma_load_3d(vs, &tmV, &full[stage], 0, key0, plane);
        tma_load_3d(vs + kTileBytes / 2, &tmV, &full[stage], 64, key0, plane);
        ++issued;
      }
      if (!ok) {
        for (int t = issued - 1; t >= 0 && t >= issued - kStages; --t)
          mbar_wait_bounded(&full[t % kStages], (uint32_t)((t / kStages) & 1), nullptr);
        raise_error(p.err, DLM_ETIMEOUT);
      }
    }
    return;
  }

  // ---------------- consumers: 16 query rows per warp ----------------
  uint32_t qf[8][4];
  {
    const int mi = lane >> 3;
    const int row = warp * 16 + (lane & 7) + (mi & 1) * 8;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int ch = 2 * ks + (mi >> 1);
      ldsm_x4(smem_u32(qs + (ch >> 3) * (kRowsCta * 128) + sw128_off(row, ch & 7)), qf[ks][0],
              qf[ks][1], qf[ks][2], qf[ks][3]);
    }
  }
  float oacc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F};
  float l_run[2] = {0.f, 0.f};

  bool ok = true;
  for (int t = 0; t < n_tiles; ++t) {
    const int stage = t % kStages;
    const uint32_t phase = (uint32_t)((t / kStages) & 1);
    if (!mbar_wait_bounded(&full[stage], phase, abort_flag)) {
      ok = false;
      break;
    }
    const uint8_t* ks = ring + stage * kStageBytes;
    const uint8_t* vs = ks + kTileBytes;

    // S = Q K^T over 64 keys
    float sc[8][4];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      sc[nb][0] = sc[nb][1] = sc[nb][2] = sc[nb][3] = 0.f;
      const int key = nb * 8 + (lane & 7);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ch = 4 * j + (lane >> 3);
        uint32_t r0, r1, r2, r3;
        ldsm_x4(smem_u32(ks + (ch >> 3) * (kTileBytes / 2) + sw128_off(key, ch & 7)), r0, r1, r2,
                r3);
        mma_bf16_16816(sc[nb], qf[2 * j], r0, r1);
        mma_bf16_16816(sc[nb], qf[2 * j + 1], r2, r3);
      }
    }
    // scale to base 2, mask keys past the end, online softmax
    const int key_base = k_begin + t * kKT;
    float mx[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = key_base + nb * 8 + 2 * (lane & 3) + (e & 1);
        const float v = (key < k_end) ? sc[nb][e] * p.scale_log2 : -CUDART_INF_F;
        sc[nb][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
    float alpha[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
      const float m_new = fmaxf(m_run[h], mx[h]);
      alpha[h] = fast_exp2(m_run[h] - m_new);
      m_run[h] = m_new;
    }
    float rsum[2] = {0.f, 0.f};
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pv = fast_exp2(sc[nb][e] - m_run[e >> 1]);
        sc[nb][e] = pv;
        rsum[e >> 1] += pv;
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) l_run[h] = l_run[h] * alpha[h] + rsum[h];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      oacc[i][0] *= alpha[0];
      oacc[i][1] *= alpha[0];
      oacc[i][2] *= alpha[1];
      oacc[i][3] *= alpha[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pf[4];
      pf[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
      pf[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
      pf[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      pf[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
      const int mi = lane >> 3;
      const int key = kk * 16 + (lane & 7) + (mi & 1) * 8;
#pragma unroll
      for (int nbp = 0; nbp < 8; ++nbp) {
        const int blk = 2 * nbp + (mi >> 1);
        uint32_t r0, r1, r2, r3;
        ldsm_x4_t(smem_u32(vs + (blk >> 3) * (kTileBytes / 2) + sw128_off(key, blk & 7)), r0, r1,
                  r2, r3);
        mma_bf16_16816(oacc[2 * nbp], pf, r0, r1);
        mma_bf16_16816(oacc[2 * nbp + 1], pf, r2, r3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  }
  if (!ok) {
    if (lane == 0) raise_error(p.err, DLM_ETIMEOUT);
    return;
  }

#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
  }
  const int rbase = rt * kRowsCta + warp * 16 + (lane >> 2);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = rbase + h * 8;
    if (r >= p.R) continue;
    if (p.nsplit == 1) {
      const int i = r / p.G, hh = r - i * p.G;
      __nv_bfloat16* dst = p.o + ((size_t)(b * p.C + i) * p.H + (g * p.G + hh)) * kDh;
      const float inv = 1.f / l_run[h];
#pragma unroll
      for (int nb = 0; nb < 16; ++nb) {
        const int dh = nb * 8 + 2 * (lane & 3);
        *reinterpret_cast<__nv_bfloat162*>(dst + dh) =
            __floats2bfloat162_rn(oacc[nb][2 * h] * inv, oacc[nb][2 * h + 1] * inv);
      }
    } else {
      const size_t slot = ((size_t)bg * p.nsplit + split) * p.R + r;
      float* dst = p.opart + slot * kDh;
#pragma unroll
      for (int nb = 0; nb < 16; ++nb) {
        const int dh = nb * 8 + 2 * (lane & 3);
        *reinterpret_cast<float2*>(dst + dh) = make_float2(oacc[nb][2 * h], oacc[nb][2 * h + 1]);
      }
      if ((lane & 3) == 0) p.ml[slot] = make_float2(m_run[h], l_run[h]);
    }
  }
}

// log-sum-exp combination of the splits of one (sequence, KV head); one warp
// per query row, lane = 4 head-dim columns.  The split weights are computed
// in parallel (lane s holds split s), then the partial rows are read in
// batches of independent loads.
__global__ void attn_combine_kernel(const float* __restrict__ opart, const float2* __restrict__ ml,
                                    __nv_bfloat16* __restrict__ o, const int32_t* __restrict__ lens,
                                    const uint8_t* __restrict__ done, const int* n_active, int H,
                                    int Hkv, int G, int C, int R, int chunk, int nsplit) {
  pdl_wait_then_release();
  if (n_active != nullptr && *n_active == 0) return;
  const int bg = blockIdx.x;
  const int b = bg / Hkv, g = bg - b * Hkv;
  if (done != nullptr && done[b]) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * (blockDim.x >> 5) + warp;
  if (r >= R) return;
  const int n_keys = lens[b] + C;
  const int nvalid = min(nsplit, (n_keys + chunk - 1) / chunk);   // <= 64
  const size_t base = (size_t)bg * nsplit * R + r;                  // slot of split s: base + s*R
  float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
  if (lane < nvalid) {
    const float2 v = ml[base + (size_t)lane * R];
    m0 = v.x;
    l0 = v.y;
  }
  if (lane + 32 < nvalid) {
    const float2 v = ml[base + (size_t)(lane + 32) * R];
    m1 = v.x;
    l1 = v.y;
  }
  float M = fmaxf(m0, m1);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float w0 = lane < nvalid ? fast_exp2(m0 - M) : 0.f;
  const float w1 = lane + 32 < nvalid ? fast_exp2(m1 - M) : 0.f;
  float L = w0 * l0 + w1 * l1;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  constexpr int kB = 8;
  for (int s0 = 0; s0 < nvalid; s0 += kB) {
    float4 x[kB];
    float w[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int sidx = s0 + u;
      const float wsel = sidx < 32 ? w0 : w1;
      w[u] = __shfl_sync(0xffffffffu, wsel, sidx & 31);
      x[u] = sidx < nvalid
                 ? *reinterpret_cast<const float4*>(opart + (base + (size_t)sidx * R) * kDh + lane * 4)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      acc[0] += w[u] * x[u].x;
      acc[1] += w[u] * x[u].y;
      acc[2] += w[u] * x[u].z;
      acc[3] += w[u] * x[u].w;
    }
  }
  const float inv = 1.f / L;
  const int i = r / G, hh = r - i * G;
  __nv_bfloat16* dst = o + ((size_t)(b * C + i) * H + (g * G + hh)) * kDh + lane * 4;
  reinterpret_cast<__nv_bfloat162*>(dst)[0] = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
  reinterpret_cast<__nv_bfloat162*>(dst)[1] = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
}

// fp32 model: one thread per query row, keys staged through shared memory
template <int DH>
__global__ void __launch_bounds__(128) attn_f32_kernel(int H, int Hkv, int C, int Lcap,
                                                       const float* __restrict__ q,
                                                       const float* __restrict__ kc,
                                                       const float* __restrict__ vc,
                                                       float* __restrict__ o,
                                                       const int32_t* __restrict__ lens,
                                                       const uint8_t* __restrict__ done,
                                                       const int* n_active, float scale) {
  pdl_wait_then_release();
  if (n_active != nullptr && *n_active == 0) return;
  constexpr int KT = 32;
  __shared__ float ks[KT][DH];
  __shared__ float vs[KT][DH];
  const int b = blockIdx.x / H, h = blockIdx.x - (blockIdx.x / H) * H;
  if (done != nullptr && done[b]) return;
  const int g = h / (H / Hkv);
  const int n_keys = lens[b] + C;
  const float* kbase = kc + ((size_t)b * Hkv + g) * Lcap * DH;
  const float* vbase = vc + ((size_t)b * Hkv + g) * Lcap * DH;
  for (int i0 = 0; i0 < C; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    const bool live = i < C;
    float qr[DH], acc[DH];
    if (live) {
      const float* qp = q + ((size_t)(b * C + i) * H + h) * DH;
#pragma unroll
      for (int d = 0; d < DH; ++d) {
        qr[d] = qp[d];
        acc[d] = 0.f;
      }
    }
    float m = -CUDART_INF_F, l = 0.f;
    for (int k0 = 0; k0 < n_keys; k0 += KT) {
      __syncthreads();
      for (int idx = threadIdx.x; idx < KT * DH; idx += blockDim.x) {
        const int kk = idx / DH, d = idx - kk * DH;
        const bool in = k0 + kk < n_keys;
        ks[kk][d] = in ? kbase[(size_t)(k0 + kk) * DH + d] : 0.f;
        vs[kk][d] = in ? vbase[(size_t)(k0 + kk) * DH + d] : 0.f;
      }
      __syncthreads();
      if (!live) continue;
      const int nk = min(KT, n_keys - k0);
      for (int kk = 0; kk < nk; ++kk) {
        float s = 0.f;
#pragma unroll
        for (int d = 0; d < DH; ++d) s = fmaf(qr[d], ks[kk][d], s);
        s *= scale;
        const float m_new = fmaxf(m, s);
        const float a = expf(m - m_new);
        const float pw = expf(s - m_new);
        l = l * a + pw;
#pragma unroll
        for (int d = 0; d < DH; ++d) acc[d] = acc[d] * a + pw * vs[kk][d];
        m = m_new;
      }
    }
    if (live) {
      float* op = o + ((size_t)(b * C + i) * H + h) * DH;
      const float inv = 1.f / l;
#pragma unroll
      for (int d = 0; d < DH; ++d) op[d] = acc[d] * inv;
    }
  }
}

}  // namespace

cudaError_t attention_bf16(const ModelDims& md, const AttnPlan& ap, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const void* q, void* o, float* opart,
                           float2* ml, const int32_t* lens, const uint8_t* done,
                           const int* n_active, int* err, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  AttnParams p;
  p.q = (const __nv_bfloat16*)q;
  p.o = (__nv_bfloat16*)o;
  p.opart = opart;
  p.ml = ml;
  p.lens = lens;
  p.done = done;
  p.n_active = n_active;
  p.err = err;
  p.H = md.H;
  p.Hkv = md.Hkv;
  p.G = ap.G;
  p.C = ap.C;
  p.R = ap.R;
  p.chunk = ap.chunk;
  p.nsplit = ap.nsplit;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)md.Dh));
  dim3 grid(ap.nsplit, ap.rtiles, ap.B * md.Hkv);
  cudaError_t e = launch_pdl(attn_bf16_kernel, grid, dim3(32 * (kWarps + 1)), kAttnSmem, st, tmK,
                             tmV, p);
  if (e != cudaSuccess || ap.nsplit == 1) return e;
  const int rows_per_block = 8;
  dim3 g2(ap.B * md.Hkv, (ap.R + rows_per_block - 1) / rows_per_block);
  return launch_pdl(attn_combine_kernel, g2, dim3(32 * rows_per_block), 0, st,
                    (const float*)opart, (const float2*)ml, (__nv_bfloat16*)o, lens, done,
                    n_active, md.H, md.Hkv, ap.G, ap.C, ap.R, ap.chunk, ap.nsplit);
}

cudaError_t attention_f32(const ModelDims& md, int B, int C, const float* q, const float* kcache,
                          const float* vcache, float* o, const int32_t* lens,
                          const uint8_t* done, const int* n_active, cudaStream_t st) {
  const float scale = (float)(1.0 / sqrt((double)md.Dh));
  const int threads = 128;
  cudaError_t e;
  if (md.Dh == 64)
    e = launch_pdl(attn_f32_kernel<64>, dim3(B * md.H), dim3(threads), 0, st, md.H, md.Hkv, C,
                   md.Lcap, q, kcache, vcache, o, lens, done, n_active, scale);
  else if (md.Dh == 128)
    e = launch_pdl(attn_f32_kernel<128>, dim3(B * md.H), dim3(threads), 0, st, md.H, md.Hkv, C,
                   md.Lcap, q, kcache, vcache, o, lens, done, n_active, scale);
  else if (md.Dh == 32)
    e = launch_pdl(attn_f32_kernel<32>, dim3(B * md.H), dim3(threads), 0, st, md.H, md.Hkv, C,
                   md.Lcap, q, kcache, vcache, o, lens, done, n_active, scale);
  else
    return cudaErrorInvalidValue;
  return e;
}

}  // namespace dlm
