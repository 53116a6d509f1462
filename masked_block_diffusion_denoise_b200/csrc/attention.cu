// Canvas attention: every canvas position of sequence b attends, with one
// joint softmax and no mask, to the cached prefix of b and all canvas
// positions (Nemotron guide, section 6: bidirectional mask over the block;
// course "Diffusion LLMs", section 14: the block reads the finished prefix
// and all of its own positions).  Canvas K/V are written by the projection
// epilogue into cache slots len..len+C-1, so the keys of sequence b are cache
// slots [0, len_b + C).
//
// bf16 kernel (tcgen05): one CTA per (key split, 128-query-row tile,
// sequence x KV head).  The query rows of a CTA are the G = H/Hkv query heads
// that share the KV head times the C canvas positions (GQA grouping), so each
// K/V tile is read once for all of them.  K and V stream from HBM with TMA;
// S = Q K^T and O += P V run on the tensor cores with S and O in tensor
// memory; the online softmax keeps one query row per thread.  The key splits
// of one (row tile, sequence x KV head) either form a thread-block cluster
// and combine their unnormalised partials through distributed shared memory
// at the end (up to 16 splits: each CTA bulk-copies to every peer the rows
// that peer combines), or write them to global memory for a second kernel
// (log-sum-exp).
#include <math_constants.h>

#include <cstdlib>
#include <cstring>

#include <cooperative_groups.h>

#include "kernels.h"

namespace dlm {

DLM_TRACE_STORAGE(attn)

namespace {

namespace cg = cooperative_groups;

constexpr int kDh = 128;
constexpr int kKeys = 128;                    // keys per tile (the N of S = Q K^T)
constexpr int kRowsCta = 128;                 // query rows per CTA (the M of both MMAs)
constexpr int kStages = 3;
constexpr int kHalf = kRowsCta * 128;         // one 64-column half of a 128-row tile: 16 KB
constexpr int kQBytes = 2 * kHalf;            // Q tile, 32 KB
constexpr int kStageBytes = 4 * kHalf;        // K and V tiles, two halves each: 64 KB
constexpr int kAttnSmem = kQBytes + kStages * kStageBytes + 1024 + 256;
constexpr uint32_t kTmemCols = 512;           // S/P double buffer (2 x 128) + O (128)
constexpr uint32_t kColO = 256;
// Online softmax with a lagging reference maximum: a row's reference moves
// to its new maximum only when that exceeds the reference by more than
// kRescaleLog2 (log2 units), so P = exp2(s - reference) stays below 2^8 and
// O is rescaled in tensor memory only when a row of the warp moves -- rarely
// after the first key tile.  Exact for any reference: the final O / l, and a
// split's (O, m, l) for the combine, do not depend on where it sat.
constexpr float kRescaleLog2 = 8.0f;

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
  int cluster;   // > 1: the nsplit CTAs of a (row tile, plane) form a cluster and combine in it
  int q_tma;     // the query tile by TMA (tmQ: q as [positions][H][Dh], box 64 x G x 128/G)
  int Lcap;      // key slots per plane in the cache
  float scale_log2;
};

// cluster exchange area (in the K/V ring, free once the last tile is done):
// this split's rows, unnormalised O (128 floats) then (max, sum) in the
// row's pad, 132 floats (528 bytes) a row; then the receive area, where
// peer j's copy of the rows this CTA combines lands at slot j.
constexpr int kXoStride = kDh + 4;
constexpr int kXoRowBytes = kXoStride * 4;
constexpr int kXoBytes = kRowsCta * kXoRowBytes;
constexpr int kMaxCluster = 16;   // 9..16: non-portable cluster sizes
constexpr int kRecvOff = kXoBytes;
static_assert(kRecvOff + (kRowsCta + kMaxCluster) * kXoRowBytes <= kStages * kStageBytes,
              "exchange areas exceed the K/V ring");
static_assert(kXoRowBytes % 16 == 0 && kRecvOff % 16 == 0, "bulk copies need 16-byte units");

// three-input maximum (sm_100 max.f32 with three operands)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// maximum of a thread's 128 scores as eight independent chains of
// three-input maxima and a tree (a single chain of 128 dependent maxima
// would be latency, not throughput)
__device__ __forceinline__ float row_max128(const float (&sv)[kKeys]) {
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fmaxf(sv[k], sv[k + 8]);
#pragma unroll
  for (int j = 16; j < kKeys; j += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = fmax3(m[k], sv[j + k], sv[j + 8 + k]);
  return fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// One CTA per (key split, 128-query-row tile, sequence x KV head), 6 warps:
//   warp 0     TMA producer: 128-key K and V tiles (two 64-column halves each,
//              128-byte swizzle) into a 3-stage ring;
//   warp 1     MMA issuer: S(t) = Q K(t)^T into TMEM buffer t % 2, issued one
//              tile ahead; then O += P(t) V(t), P read from TMEM (bf16 pairs
//              written over S(t)), V as an MN-major shared-memory operand;
//   warps 2-5  softmax: thread = query row = TMEM lane; reads S(t), keeps the
//              running max and sum (base 2), writes P(t) to TMEM and, only
//              when a row's maximum moved, rescales O in TMEM.
// tcgen05 operations of the issuing thread run in order, so S(t+2) cannot
// overwrite P(t) before P(t) V(t) has read it.
template <bool POLY>
__global__ void __launch_bounds__(192, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmQ, const AttnParams p) {
  // timeline marks: 2 wait returned, 3 query and first K/V tile in shared
  // memory, 4 O complete, 5 cluster barrier passed, 6 peers' rows received,
  // 7 combined
  DLM_TRACE_CTA(TRACE_ATTENTION);
  // Before the wait for the previous kernel this CTA reads only data of
  // kernels that finished before that one started (cache lengths, done
  // flags, the active count; read through L2, where no stale copy can be
  // left) and the cached prefix: barriers, tensor memory and the K/V tiles
  // that lie wholly inside the prefix are set up early; the query tile and
  // tiles that reach the canvas slots follow the wait.
  const int split = blockIdx.x, rt = blockIdx.y, bg = blockIdx.z;
  const int b = bg / p.Hkv, g = bg - b * p.Hkv;
  const int na = p.n_active != nullptr ? __ldcg(p.n_active) : 1;
  const bool dn = p.done != nullptr && __ldcg(p.done + b) != 0;
  const int len_b = __ldcg(p.lens + b);
  if (na == 0 || dn) return;
  const int n_keys = len_b + p.C;
  // a cluster's CTAs share the plane, so this exit is uniform over a cluster
  if (!DLM_IN_BOUNDS(n_keys - 1, p.Lcap, p.err)) return;
  const int k_begin = split * p.chunk;
  // a split past the keys exits at once, except in a cluster, where it still
  // takes part in the exchange (with no rows of its own)
  if (k_begin >= n_keys && p.cluster <= 1) return;
  const int k_end = min(k_begin + p.chunk, n_keys);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + kKeys - 1) / kKeys : 0;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qs = smem;
  uint8_t* ring = smem + kQBytes;
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(ring + kStages * kStageBytes);
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;   // [2]: S(t) in TMEM buffer t % 2
  // [2]: P(t) in TMEM buffer t % 2.  One barrier per buffer keeps the softmax
  // at most one phase ahead of the issuer: it can arrive for t + 2 only after
  // S(t + 2), which is issued after P(t) V(t)
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* mma_done = pv_done + 1;
  uint64_t* q_full = mma_done + 1;
  uint64_t* rx = q_full + 1;   // cluster exchange: the peers' rows have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rx + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
    }
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    mbar_init(q_full, 1);
    mbar_init(rx, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  __syncthreads();
  const int plane = b * p.Hkv + g;
  auto issue_kv = [&](int t) {
    const int st = t % kStages;
    uint8_t* base = ring + st * kStageBytes;
    const int key0 = k_begin + t * kKeys;
    mbar_arrive_expect_tx(&kv_full[st], kStageBytes);
    tma_load_3d(base, &tmK, &kv_full[st], 0, key0, plane);
    tma_load_3d(base + kHalf, &tmK, &kv_full[st], 64, key0, plane);
    tma_load_3d(base + 2 * kHalf, &tmV, &kv_full[st], 0, key0, plane);
    tma_load_3d(base + 3 * kHalf, &tmV, &kv_full[st], 64, key0, plane);
  };
  int pre = 0;   // tiles issued before the wait (prefix keys only)
  const bool q_by_tma = p.q_tma != 0 && n_tiles > 0;   // a split without keys needs no query
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmK);
    tma_prefetch(&tmV);
    if (q_by_tma) tma_prefetch(&tmQ);
    const int n_prefix = len_b;
    while (pre < kStages && pre < n_tiles && k_begin + (pre + 1) * kKeys <= n_prefix) {
      issue_kv(pre);
      ++pre;
    }
  }
  pdl_wait_then_release();
  if (tid == 0) DLM_TRACE_MARK(2);
  if (q_by_tma) {
    // the query tile: positions b*C + rt*128/G .., the G heads of KV head g,
    // two 64-column halves with the 128-byte swizzle; rows past R (the next
    // canvas's positions, or zero fill past the buffer) are never stored
    if (warp == 0 && lane == 0) {
      const int z0 = b * p.C + rt * (kRowsCta / p.G);
      mbar_arrive_expect_tx(q_full, kQBytes);
      tma_load_3d(qs, &tmQ, q_full, 0, g * p.G, z0);
      tma_load_3d(qs + kHalf, &tmQ, q_full, 64, g * p.G, z0);
    }
  } else {
    // query tile -> shared memory, two 64-column halves, 128-byte swizzle;
    // every load of a thread is issued before the first store

    constexpr int kQChunks = kRowsCta * 16;                  // 16-byte chunks
    constexpr int kPer = (kQChunks + 191) / 192;             // per thread at 192 threads
    uint4 val[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = tid + u * 192;
      const int lr = idx >> 4, ch = idx & 15;
      const int r = rt * kRowsCta + lr;
      val[u] = make_uint4(0, 0, 0, 0);
      if (idx < kQChunks && r < p.R) {
        const int i = r / p.G, hh = r - i * p.G;
        val[u] = *reinterpret_cast<const uint4*>(
            p.q + ((size_t)(b * p.C + i) * p.H + (g * p.G + hh)) * kDh + ch * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = tid + u * 192;
      if (idx < kQChunks) {
        const int lr = idx >> 4, ch = idx & 15;
        *reinterpret_cast<uint4*>(qs + (ch >> 3) * kHalf + sw128_off(lr, ch & 7)) = val[u];
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = pre;
      for (int t = pre; t < n_tiles; ++t) {
        const int st = t % kStages;
        if (!mbar_wait_bounded(&kv_empty[st], (uint32_t)(((t / kStages) & 1) ^ 1), abort_flag))
          break;
        issue_kv(t);
        ++issued;
      }
      if (*abort_flag) {
        // let the copies already in flight land before the CTA exits
        for (int t = issued - 1; t >= 0 && t >= issued - kStages; --t)
          mbar_wait_bounded(&kv_full[t % kStages], (uint32_t)((t / kStages) & 1), nullptr);
      }
      if (q_by_tma) mbar_wait_bounded(q_full, 0, nullptr);   // the query tile has landed
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kRowsCta, kKeys);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kRowsCta, kDh, true);
      const uint32_t qaddr = smem_u32(qs);
      auto issue_s = [&](int t) {
        const uint32_t kaddr = smem_u32(ring + (t % kStages) * kStageBytes);
        const uint32_t d = tmem_base + (uint32_t)((t & 1) * kKeys);
#pragma unroll
        for (int k = 0; k < kDh / 16; ++k) {
          const uint32_t off = (uint32_t)((k >> 2) * kHalf + (k & 3) * 32);
          umma_bf16(d, sw128_desc(qaddr + off), sw128_desc(kaddr + off), idesc_s, k > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[t & 1]);
      };
      bool ok = n_tiles > 0 && (!q_by_tma || mbar_wait_bounded(q_full, 0, abort_flag)) &&
                mbar_wait_bounded(&kv_full[0], 0, abort_flag);
      DLM_TRACE_MARK(3);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int t = 0; ok && t < n_tiles; ++t) {
        if (t + 1 < n_tiles) {
          const int t1 = t + 1;
          if (!mbar_wait_bounded(&kv_full[t1 % kStages], (uint32_t)((t1 / kStages) & 1),
                                 abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(t1);
        }
        if (!mbar_wait_bounded(&p_full[t & 1], (uint32_t)((t >> 1) & 1), abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t vaddr = smem_u32(ring + (t % kStages) * kStageBytes + 2 * kHalf);
        const uint32_t pcol = tmem_base + (uint32_t)((t & 1) * kKeys);
#pragma unroll
        for (int k = 0; k < kKeys / 16; ++k) {
          const uint64_t bdesc = sw128_desc_mn(vaddr + (uint32_t)(k * 2048), kHalf);
          umma_bf16_tmem_a(tmem_base + kColO, pcol + (uint32_t)(k * 8), bdesc, idesc_o,
                           (t > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(pv_done);
        umma_commit(&kv_empty[t % kStages]);
      }
      umma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr);
    }
  } else {
    // ---------------- softmax warps ----------------
    const int quad = warp & 3;
    const int row = quad * 32 + lane;                 // query row within the tile = TMEM lane
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quad * 32) << 16);
    float m_run = -CUDART_INF_F, l_run = 0.f;
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int buf = t & 1;
      if (!mbar_wait_bounded(&s_full[buf], (uint32_t)((t >> 1) & 1), abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[kKeys];
      {
        uint32_t raw[kKeys / 32][32];
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c)
          tmem_ld32_nowait(lane_addr + (uint32_t)(buf * kKeys + c * 32), raw[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j) sv[c * 32 + j] = __uint_as_float(raw[c][j]);
      }
      const int key_base = k_begin + t * kKeys;
      if (key_base + kKeys > k_end) {   // ragged last tile (warp-uniform): mask past the end
#pragma unroll
        for (int j = 0; j < kKeys; ++j)
          if (key_base + j >= k_end) sv[j] = -CUDART_INF_F;
      }
      // maximum on the raw scores (the scale is positive), then one FFMA per score
      const float mx = row_max128(sv) * p.scale_log2;
      const bool move = __any_sync(0xffffffffu, mx > m_run + kRescaleLog2);
      const float m_new = move ? fmaxf(m_run, mx) : m_run;
      const float alpha = move ? fast_exp2(m_run - m_new) : 1.f;
      // eight independent partial sums (no 128-long dependency chain)
      // POLY: 3 of every 8 exponentials on the FMA pipe (exp2_poly), the
      // rest on the exponential unit
      float rs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < kKeys; ++j) {
        const float x = fmaf(sv[j], p.scale_log2, -m_new);
        const float e = POLY && (j & 7) >= 5 ? exp2_poly(x) : fast_exp2(x);
        sv[j] = e;
        rs[j & 7] += e;
      }
      const float rsum = ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
      l_run = l_run * alpha + rsum;
      m_run = m_new;
      // P(t) in bf16, two keys per 32-bit TMEM column, over the S(t) columns
#pragma unroll
      for (int c = 0; c < kKeys / 64; ++c) {
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) w[j] = pack_bf16(sv[64 * c + 2 * j], sv[64 * c + 2 * j + 1]);
        tmem_st32_u(lane_addr + (uint32_t)(buf * kKeys + c * 32), w);
      }
      // rescale O only when the warp's reference moved; O must first hold
      // every earlier P V
      if (t > 0 && move) {
        if (!mbar_wait_bounded(pv_done, (uint32_t)((t - 1) & 1), abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kDh / 32; ++c) {
          float o[32];
          tmem_ld32(lane_addr + kColO + (uint32_t)(c * 32), o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] *= alpha;
          tmem_st32(lane_addr + kColO + (uint32_t)(c * 32), o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[buf]);
    }
    // every MMA has completed (a one-phase barrier: no parity can alias, as
    // a wait on pv_done for the last tile could while P(t-1) V(t-1) runs)
    float ov[kDh];
    bool have = false;
    if (ok && n_tiles > 0 && mbar_wait_bounded(mma_done, 0, abort_flag)) {
      tc_fence_after();
      have = true;
      if (row == 0) DLM_TRACE_MARK(4);
      {
        uint32_t raw[kDh / 32][32];
#pragma unroll
        for (int c = 0; c < kDh / 32; ++c)
          tmem_ld32_nowait(lane_addr + kColO + (uint32_t)(c * 32), raw[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kDh / 32; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[c * 32 + j] = __uint_as_float(raw[c][j]);
      }
    }
    if (p.cluster > 1) {
      // this split's rows for the cluster: unnormalised O, running max and sum
      fence_proxy_async_smem();
      // 16-byte stores: a warp's rows (528 bytes apart) fill all 32 banks
      float4* xo = reinterpret_cast<float4*>(ring + row * kXoRowBytes);
#pragma unroll
      for (int c = 0; c < kDh / 4; ++c)
        xo[c] = have ? make_float4(ov[4 * c], ov[4 * c + 1], ov[4 * c + 2], ov[4 * c + 3])
                     : make_float4(0.f, 0.f, 0.f, 0.f);
      xo[kDh / 4] = have ? make_float4(m_run, l_run, 0.f, 0.f)
                         : make_float4(-CUDART_INF_F, 0.f, 0.f, 0.f);
      fence_proxy_async_smem();   // the rows are read by bulk copies (async proxy)
    } else if (have) {
      const int r = rt * kRowsCta + row;
      if (r < p.R) {
        if (p.nsplit == 1) {
          const int i = r / p.G, hh = r - i * p.G;
          __nv_bfloat16* dst = p.o + ((size_t)(b * p.C + i) * p.H + (g * p.G + hh)) * kDh;
          const float inv = 1.f / l_run;
#pragma unroll
          for (int c = 0; c < kDh / 8; ++c) {
            uint4 w;
            w.x = pack_bf16(ov[8 * c + 0] * inv, ov[8 * c + 1] * inv);
            w.y = pack_bf16(ov[8 * c + 2] * inv, ov[8 * c + 3] * inv);
            w.z = pack_bf16(ov[8 * c + 4] * inv, ov[8 * c + 5] * inv);
            w.w = pack_bf16(ov[8 * c + 6] * inv, ov[8 * c + 7] * inv);
            reinterpret_cast<uint4*>(dst)[c] = w;
          }
        } else {
          const size_t slot = ((size_t)bg * p.nsplit + split) * p.R + r;
          float4* dst = reinterpret_cast<float4*>(p.opart + slot * kDh);
#pragma unroll
          for (int c = 0; c < kDh / 4; ++c)
            dst[c] = make_float4(ov[4 * c], ov[4 * c + 1], ov[4 * c + 2], ov[4 * c + 3]);
          p.ml[slot] = make_float2(m_run, l_run);
        }
      }
    }
  }

  if (p.cluster > 1) {
    // every split's rows are in its shared memory; CTA q of the cluster
    // combines rows q*ceil(128/n) .. of the tile for all splits (fixed order).
    cg::cluster_group cluster = cg::this_cluster();
    const int n = p.cluster;
    const int q = (int)cluster.block_rank();
    const int per = (kRowsCta + n - 1) / n;
    const int r0 = min(kRowsCta, q * per), r1 = min(kRowsCta, r0 + per);
    uint8_t* recv = ring + kRecvOff;
    // every CTA copies, with one bulk copy per peer, the rows that peer
    // combines into the peer's receive area; then each CTA combines from
    // its own shared memory
    if (tid == 0) mbar_arrive_expect_tx(rx, (uint32_t)((n - 1) * (r1 - r0) * kXoRowBytes));
    cluster.sync();   // rows written, receive barriers armed
    if (tid == 0) DLM_TRACE_MARK(5);
    if (tid < n && tid != q) {
      const int a0 = min(kRowsCta, tid * per), a1 = min(kRowsCta, a0 + per);
      if (a1 > a0)
        bulk_copy_to_peer(cluster_addr(smem_u32(recv + q * per * kXoRowBytes), tid),
                          smem_u32(ring + a0 * kXoRowBytes), (uint32_t)((a1 - a0) * kXoRowBytes),
                          cluster_addr(smem_u32(rx), tid));
    }
    // the copies into this CTA land before it reads them -- or, after an
    // abort, before it exits
    if (!mbar_wait_bounded(rx, 0, abort_flag)) mbar_wait_bounded(rx, 0, nullptr);
    if (tid == 0) DLM_TRACE_MARK(6);
    const float* xo_p[kMaxCluster];   // split j's row r0 + i: xo_p[j] + i * kXoStride
#pragma unroll
    for (int j = 0; j < kMaxCluster; ++j)
      xo_p[j] = j == q ? reinterpret_cast<const float*>(ring + r0 * kXoRowBytes)
                       : reinterpret_cast<const float*>(recv + (j < n ? j : 0) * per * kXoRowBytes);
    for (int it = tid; it < (r1 - r0) * (kDh / 4); it += blockDim.x) {
      const int lr = r0 + it / (kDh / 4);
      const int c4 = (it % (kDh / 4)) * 4;
      const int r = rt * kRowsCta + lr;
      if (r >= p.R) continue;
      float2 ml[kMaxCluster];
      float4 ov4[kMaxCluster];
#pragma unroll
      for (int j = 0; j < kMaxCluster; ++j) {
        const float* src = xo_p[j] + (lr - r0) * kXoStride;
        ml[j] = j < n ? *reinterpret_cast<const float2*>(src + kDh) : make_float2(-CUDART_INF_F, 0.f);
        ov4[j] = j < n ? *reinterpret_cast<const float4*>(src + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float M = -CUDART_INF_F;
#pragma unroll
      for (int j = 0; j < kMaxCluster; ++j) M = fmaxf(M, ml[j].x);
      float L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < kMaxCluster; ++j) {
        const float w = ml[j].x == -CUDART_INF_F ? 0.f : fast_exp2(ml[j].x - M);
        L = fmaf(w, ml[j].y, L);
        acc.x = fmaf(w, ov4[j].x, acc.x);
        acc.y = fmaf(w, ov4[j].y, acc.y);
        acc.z = fmaf(w, ov4[j].z, acc.z);
        acc.w = fmaf(w, ov4[j].w, acc.w);
      }
      const float inv = 1.f / L;
      const int i = r / p.G, hh = r - i * p.G;
      __nv_bfloat16* dst = p.o + ((size_t)(b * p.C + i) * p.H + (g * p.G + hh)) * kDh + c4;
      uint2 w2;
      w2.x = pack_bf16(acc.x * inv, acc.y * inv);
      w2.y = pack_bf16(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(dst) = w2;
    }
    if (tid == 0) DLM_TRACE_MARK(7);
    // every copy into every CTA of the cluster has landed (each CTA arrives
    // after its receive barrier): the rows may be released
    cluster.sync();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (tid == 0 && *abort_flag) raise_error(p.err, DLM_ETIMEOUT);
}

// ---------------------------------------------------------------------------
// Two query-row tiles per CTA (256 rows): when a KV head has at least 256
// query rows (G * C >= 256), one CTA takes two 128-row tiles of the same
// (sequence, KV head, key split), so each K/V tile is brought in once for
// both and the two softmax warpgroups keep the exponent units busy while
// the tensor core works for the other.  12 warps in three warpgroups:
//   warps 0-3  softmax of row tile 0, warps 4-7 of row tile 1: thread =
//              query row = TMEM lane; the 128 scores of a key tile are read
//              from tensor memory once and kept in registers (the warpgroups
//              raise their register limit to 224, setmaxnreg);
//   warp 8     TMA producer: K tiles into a 2-slot ring, V tiles into a
//              3-slot ring (128 keys x 128 dims, two 64-column halves each);
//   warp 9     MMA issuer, polling without blocking: for each row tile i it
//              issues O_i += P_i(t) V(t) as soon as P_i(t) and V(t) are there
//              and S_i(t+1) = Q_i K(t+1)^T right after (one S buffer per row
//              tile: tcgen05 operations of one thread run in order, so S_i(t+1)
//              is written after P_i(t) has been read, and once S_i(t+1) is
//              complete O_i holds every earlier P_i V, which the softmax may
//              then rescale); a row tile never waits for the other;
//   warps 10-11 idle (they complete the third warpgroup for setmaxnreg).
// TMEM: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).  Splits write
// bf16 O (one split) or f32 partials for attn_combine_kernel.
// ---------------------------------------------------------------------------
constexpr int kTile2 = 2 * kHalf;                 // one 128-row / 128-key tile: 32 KB
constexpr int kKSlots2 = 2, kVSlots2 = 3;
constexpr int kAttn2Threads = 384;
constexpr int kAttn2Smem = 2 * kTile2 + (kKSlots2 + kVSlots2) * kTile2 + 1024 + 512;
static_assert(kAttn2Smem <= 232448, "two-tile attention exceeds shared memory");
// register split: 384 threads launch with 168 registers each (64512); the
// third warpgroup gives back 112 per thread, the softmax warpgroups take 56
constexpr int kAttn2RegsSoftmax = 224, kAttn2RegsOther = 56;
static_assert(kAttn2RegsSoftmax * 256 + kAttn2RegsOther * 128 <= 168 * kAttn2Threads,
              "register split exceeds the launch's registers");

template <bool POLY>
__global__ void __launch_bounds__(kAttn2Threads, 1)
    attn_tc2_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmQ, const AttnParams p) {
  // timeline marks: 2 wait returned, 3 query and first K tile in shared
  // memory, 4 O complete, 5 row tile 0's softmax of key tile 1 begins, 6 its
  // last key tile's P is written, 7 the producer has issued its last tile
  DLM_TRACE_CTA(TRACE_ATTENTION);
  const int split = blockIdx.x, pair = blockIdx.y, bg = blockIdx.z;
  const int b = bg / p.Hkv, g = bg - b * p.Hkv;
  const int na = p.n_active != nullptr ? __ldcg(p.n_active) : 1;
  const bool dn = p.done != nullptr && __ldcg(p.done + b) != 0;
  const int len_b = __ldcg(p.lens + b);
  if (na == 0 || dn) return;
  const int n_keys = len_b + p.C;
  if (!DLM_IN_BOUNDS(n_keys - 1, p.Lcap, p.err)) return;
  const int k_begin = split * p.chunk;
  if (k_begin >= n_keys) return;
  const int k_end = min(k_begin + p.chunk, n_keys);
  const int n_tiles = (k_end - k_begin + kKeys - 1) / kKeys;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qs = smem;                                   // Q0, Q1
  uint8_t* kring = smem + 2 * kTile2;
  uint8_t* vring = kring + kKSlots2 * kTile2;
  uint64_t* k_full = reinterpret_cast<uint64_t*>(vring + kVSlots2 * kTile2);
  uint64_t* k_empty = k_full + kKSlots2;
  uint64_t* v_full = k_empty + kKSlots2;
  uint64_t* v_empty = v_full + kVSlots2;
  uint64_t* s_full = v_empty + kVSlots2;                // [2]
  uint64_t* p_full = s_full + 2;                        // [2]
  uint64_t* o_done = p_full + 2;
  uint64_t* q_full = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kProducer = 8, kMma = 9;
  if (tid == 0) {
    for (int i = 0; i < kKSlots2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kVSlots2; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
    }
    mbar_init(o_done, 1);
    mbar_init(q_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMma) tmem_alloc(tmem_slot, kTmemCols);
  __syncthreads();
  const int plane = b * p.Hkv + g;
  auto issue_k = [&](int t) {
    uint8_t* base = kring + (t % kKSlots2) * kTile2;
    const int key0 = k_begin + t * kKeys;
    mbar_arrive_expect_tx(&k_full[t % kKSlots2], kTile2);
    tma_load_3d(base, &tmK, &k_full[t % kKSlots2], 0, key0, plane);
    tma_load_3d(base + kHalf, &tmK, &k_full[t % kKSlots2], 64, key0, plane);
  };
  auto issue_v = [&](int t) {
    uint8_t* base = vring + (t % kVSlots2) * kTile2;
    const int key0 = k_begin + t * kKeys;
    mbar_arrive_expect_tx(&v_full[t % kVSlots2], kTile2);
    tma_load_3d(base, &tmV, &v_full[t % kVSlots2], 0, key0, plane);
    tma_load_3d(base + kHalf, &tmV, &v_full[t % kVSlots2], 64, key0, plane);
  };
  // K/V tiles wholly inside the cached prefix do not depend on the previous
  // kernel: the first ring slots' worth are issued before the wait
  int pre = 0;
  if (warp == kProducer && lane == 0) {
    tma_prefetch(&tmK);
    tma_prefetch(&tmV);
    if (p.q_tma) tma_prefetch(&tmQ);
    while (pre < kKSlots2 && pre < n_tiles && k_begin + (pre + 1) * kKeys <= len_b) {
      issue_k(pre);
      issue_v(pre);
      ++pre;
    }
  }
  pdl_wait_then_release();
  if (tid == 0) DLM_TRACE_MARK(2);
  const int row_base = pair * 2 * kRowsCta;   // first query row of tile 0
  if (p.q_tma) {
    if (warp == kProducer && lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * kTile2);
      for (int i = 0; i < 2; ++i) {
        const int z0 = b * p.C + (row_base + i * kRowsCta) / p.G;
        tma_load_3d(qs + i * kTile2, &tmQ, q_full, 0, g * p.G, z0);
        tma_load_3d(qs + i * kTile2 + kHalf, &tmQ, q_full, 64, g * p.G, z0);
      }
    }
  } else {
    // plain loads: 256 rows x 16 chunks of 16 bytes, rows past R zero
    for (int idx = tid; idx < 2 * kRowsCta * 16; idx += blockDim.x) {
      const int lr = idx >> 4, ch = idx & 15;
      const int r = row_base + lr;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (r < p.R) {
        const int i = r / p.G, hh = r - i * p.G;
        val = *reinterpret_cast<const uint4*>(
            p.q + ((size_t)(b * p.C + i) * p.H + (g * p.G + hh)) * kDh + ch * 8);
      }
      const int tl = lr >> 7, tr = lr & 127;
      *reinterpret_cast<uint4*>(qs + tl * kTile2 + (ch >> 3) * kHalf + sw128_off(tr, ch & 7)) =
          val;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the register split heads each warpgroup's branch (every warp of the
  // warpgroup executes it)
  if (warp >= kProducer) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kAttn2RegsOther));
  if (warp == kProducer) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = pre;
      for (int t = pre; t < n_tiles; ++t) {
        if (t >= kKSlots2 &&
            !mbar_wait_bounded(&k_empty[t % kKSlots2], (uint32_t)(((t / kKSlots2) & 1) ^ 1),
                               abort_flag))
          break;
        if (t >= kVSlots2 &&
            !mbar_wait_bounded(&v_empty[t % kVSlots2], (uint32_t)(((t / kVSlots2) & 1) ^ 1),
                               abort_flag))
          break;   // K(t) is not issued either: the K and V counts stay equal
        issue_k(t);
        issue_v(t);
        ++issued;
      }
      DLM_TRACE_MARK(7);
      if (*abort_flag) {
        // let the copies already in flight land before the CTA exits
        for (int t = issued - 1; t >= 0 && t >= issued - kKSlots2; --t)
          mbar_wait_bounded(&k_full[t % kKSlots2], (uint32_t)((t / kKSlots2) & 1), nullptr);
        for (int t = issued - 1; t >= 0 && t >= issued - kVSlots2; --t)
          mbar_wait_bounded(&v_full[t % kVSlots2], (uint32_t)((t / kVSlots2) & 1), nullptr);
      }
      if (p.q_tma) mbar_wait_bounded(q_full, 0, nullptr);   // the query tiles have landed
    }
  } else if (warp == kMma) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kRowsCta, kKeys);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kRowsCta, kDh, true);
      auto issue_s = [&](int i, int t) {
        const uint32_t qaddr = smem_u32(qs + i * kTile2);
        const uint32_t kaddr = smem_u32(kring + (t % kKSlots2) * kTile2);
        const uint32_t d = tmem_base + (uint32_t)(i * kKeys);
#pragma unroll
        for (int k = 0; k < kDh / 16; ++k) {
          const uint32_t off = (uint32_t)((k >> 2) * kHalf + (k & 3) * 32);
          umma_bf16(d, sw128_desc(qaddr + off), sw128_desc(kaddr + off), idesc_s, k > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[i]);
      };
      auto issue_pv = [&](int i, int t) {
        const uint32_t vaddr = smem_u32(vring + (t % kVSlots2) * kTile2);
        const uint32_t pcol = tmem_base + (uint32_t)(i * kKeys);
        const uint32_t ocol = tmem_base + kColO + (uint32_t)(i * kDh);
#pragma unroll
        for (int k = 0; k < kKeys / 16; ++k) {
          const uint64_t bdesc = sw128_desc_mn(vaddr + (uint32_t)(k * 2048), kHalf);
          umma_bf16_tmem_a(ocol, pcol + (uint32_t)(k * 8), bdesc, idesc_o,
                           (t > 0 || k > 0) ? 1u : 0u);
        }
      };
      // s_next[i]: next S tile of row tile i; pv_next[i]: next P V tile.
      // S_i(t) may be issued once P_i(t-1) V has been (s_next == pv_next);
      // a K slot is released when both row tiles' S of it are issued, a V
      // slot when both P V are.  A row tile is at most one phase ahead of
      // any barrier it tests (its S(t) needs its S(t-2), whose K slot phase
      // came first; its P V(t) needs the V slot's previous phase done), so
      // the non-blocking parity tests cannot alias.
      int s_next[2] = {0, 0}, pv_next[2] = {0, 0};
      bool ok = !p.q_tma || mbar_wait_bounded(q_full, 0, abort_flag);
      uint64_t t_idle = 0;
      for (uint32_t spin = 0; ok && (pv_next[0] < n_tiles || pv_next[1] < n_tiles); ++spin) {
        bool progress = false;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int ts = s_next[i];
          if (ts < n_tiles && ts == pv_next[i] &&
              mbar_test_wait(&k_full[ts % kKSlots2], (uint32_t)((ts / kKSlots2) & 1))) {
            if (ts == 0 && i == 0) DLM_TRACE_MARK(3);
            tc_fence_after();
            issue_s(i, ts);
            s_next[i] = ts + 1;
            progress = true;
            // K(ts) is free once both row tiles' S(ts) have been issued
            if (s_next[0] > ts && s_next[1] > ts) umma_commit(&k_empty[ts % kKSlots2]);
          }
          const int tp = pv_next[i];
          if (tp < s_next[i] && mbar_test_wait(&p_full[i], (uint32_t)(tp & 1)) &&
              mbar_test_wait(&v_full[tp % kVSlots2], (uint32_t)((tp / kVSlots2) & 1))) {
            tc_fence_after();
            issue_pv(i, tp);
            pv_next[i] = tp + 1;
            progress = true;
            if (pv_next[0] > tp && pv_next[1] > tp) umma_commit(&v_empty[tp % kVSlots2]);
          }
        }
        if (!progress) {
          // nothing ready: sleep on the row tile that has waited longest for
          // its P (briefly, so the other one is not kept waiting), instead of
          // spinning on the issue slots the softmax warps of this SM
          // sub-partition need
          const int w = pv_next[0] <= pv_next[1] ? 0 : 1;
          if (pv_next[w] < s_next[w])
            mbar_try_wait_hint(&p_full[w], (uint32_t)(pv_next[w] & 1), 200u);
        }
        if (progress) {
          t_idle = 0;
        } else if ((spin & 255u) == 0) {
          if (*abort_flag) break;
          const uint64_t now = global_ns();
          if (t_idle == 0) {
            t_idle = now;
          } else if (now - t_idle > kWaitLimitNs) {
            *abort_flag = 1;
            break;
          }
        }
      }
      // O complete (or, after an abort, every MMA issued has finished)
      umma_commit(o_done);
      mbar_wait_bounded(o_done, 0, nullptr);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kAttn2RegsSoftmax));
    // ---------------- softmax warpgroups ----------------
    const int tile = warp >> 2;                       // row tile of this warpgroup
    const int quad = warp & 3;
    const int row = quad * 32 + lane;                 // row within the tile = TMEM lane
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quad * 32) << 16);
    const uint32_t s_col = (uint32_t)(tile * kKeys);
    const uint32_t o_col = kColO + (uint32_t)(tile * kDh);
    float m_run = -CUDART_INF_F, l_run = 0.f;
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      if (!mbar_wait_bounded(&s_full[tile], (uint32_t)(t & 1), abort_flag)) {
        ok = false;
        break;
      }
      if (t == 1 && tile == 0 && row == 0) DLM_TRACE_MARK(5);
      tc_fence_after();
      float sv[kKeys];
      {
        uint32_t raw[kKeys / 32][32];
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c)
          tmem_ld32_nowait(lane_addr + s_col + (uint32_t)(c * 32), raw[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j) sv[c * 32 + j] = __uint_as_float(raw[c][j]);
      }
      const int key_base = k_begin + t * kKeys;
      if (key_base + kKeys > k_end) {   // ragged last tile (warp-uniform): mask past the end
#pragma unroll
        for (int j = 0; j < kKeys; ++j)
          if (key_base + j >= k_end) sv[j] = -CUDART_INF_F;
      }
      const float mx = row_max128(sv) * p.scale_log2;
      const bool move = __any_sync(0xffffffffu, mx > m_run + kRescaleLog2);
      const float m_new = move ? fmaxf(m_run, mx) : m_run;
      const float alpha = move ? fast_exp2(m_run - m_new) : 1.f;
      // eight independent partial sums (no 128-long dependency chain)
      float rs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kKeys / 32; ++c) {
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          // POLY: pairs 10..15 of every 16 (3 in 8 exponentials) on the FMA pipe
          const float x0 = fmaf(sv[32 * c + 2 * j], p.scale_log2, -m_new);
          const float x1 = fmaf(sv[32 * c + 2 * j + 1], p.scale_log2, -m_new);
          const float e0 = POLY && j >= 10 ? exp2_poly(x0) : fast_exp2(x0);
          const float e1 = POLY && j >= 10 ? exp2_poly(x1) : fast_exp2(x1);
          rs[j & 7] += e0 + e1;
          w[j] = pack_bf16(e0, e1);
        }
        tmem_st16_u(lane_addr + s_col + (uint32_t)(c * 16), w);
      }
      const float rsum = ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
      l_run = l_run * alpha + rsum;
      m_run = m_new;
      // O_i holds every earlier P_i V (see the MMA issuer): rescale it only
      // when the warp's reference moved
      if (t > 0 && move) {
#pragma unroll
        for (int c = 0; c < kDh / 32; ++c) {
          float o[32];
          tmem_ld32(lane_addr + o_col + (uint32_t)(c * 32), o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] *= alpha;
          tmem_st32(lane_addr + o_col + (uint32_t)(c * 32), o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[tile]);
      if (t == n_tiles - 1 && tile == 0 && row == 0) DLM_TRACE_MARK(6);
    }
    if (ok && mbar_wait_bounded(o_done, 0, abort_flag)) {
      tc_fence_after();
      if (row == 0 && tile == 0) DLM_TRACE_MARK(4);
      // O in chunks of 32 columns: bf16 rows (one split) or f32 partials
      const int r = row_base + tile * kRowsCta + row;
      const bool live = r < p.R;
      const int i = r / p.G, hh = r - i * p.G;
      __nv_bfloat16* dst = p.o + ((size_t)(b * p.C + i) * p.H + (g * p.G + hh)) * kDh;
      const size_t slot = ((size_t)bg * p.nsplit + split) * p.R + r;
      const float inv = 1.f / l_run;
#pragma unroll 1
      for (int c = 0; c < kDh / 32; ++c) {
        float ov[32];
        tmem_ld32(lane_addr + o_col + (uint32_t)(c * 32), ov);
        if (!live) continue;
        if (p.nsplit == 1) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 w;
            w.x = pack_bf16(ov[8 * q4 + 0] * inv, ov[8 * q4 + 1] * inv);
            w.y = pack_bf16(ov[8 * q4 + 2] * inv, ov[8 * q4 + 3] * inv);
            w.z = pack_bf16(ov[8 * q4 + 4] * inv, ov[8 * q4 + 5] * inv);
            w.w = pack_bf16(ov[8 * q4 + 6] * inv, ov[8 * q4 + 7] * inv);
            reinterpret_cast<uint4*>(dst + c * 32)[q4] = w;
          }
        } else {
          float4* pd = reinterpret_cast<float4*>(p.opart + slot * kDh + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            pd[q4] = make_float4(ov[4 * q4], ov[4 * q4 + 1], ov[4 * q4 + 2], ov[4 * q4 + 3]);
        }
      }
      if (live && p.nsplit > 1) p.ml[slot] = make_float2(m_run, l_run);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (tid == 0 && *abort_flag) raise_error(p.err, DLM_ETIMEOUT);
}

// log-sum-exp combination of the splits of one (sequence, KV head); one warp
// per query row, lane = 4 head-dim columns.  The split weights are computed
// in parallel (lane s holds split s), then the partial rows are read in
// batches of independent loads.
__global__ void attn_combine_kernel(const float* __restrict__ opart, const float2* __restrict__ ml,
                                    __nv_bfloat16* __restrict__ o, const int32_t* __restrict__ lens,
                                    const uint8_t* __restrict__ done, const int* n_active, int H,
                                    int Hkv, int G, int C, int R, int chunk, int nsplit) {
  DLM_TRACE_CTA(TRACE_ATTN_COMBINE);
  pdl_wait_then_release();
  if (threadIdx.x == 0) DLM_TRACE_MARK(2);
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
                                                       const int* n_active, float scale,
                                                       int* err) {
  pdl_wait_then_release();
  if (n_active != nullptr && *n_active == 0) return;
  constexpr int KT = 32;
  __shared__ float ks[KT][DH];
  __shared__ float vs[KT][DH];
  const int b = blockIdx.x / H, h = blockIdx.x - (blockIdx.x / H) * H;
  if (done != nullptr && done[b]) return;
  const int g = h / (H / Hkv);
  const int n_keys = lens[b] + C;
  if (!DLM_IN_BOUNDS(n_keys - 1, Lcap, err)) return;
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

// diagnostic switch: DLM_ATTN_POLY=1 computes 3 of every 8 of the softmax's
// exponentials with exp2_poly on the FMA pipe instead of the exponential unit
bool attn_poly() {
  const char* e = std::getenv("DLM_ATTN_POLY");
  return e != nullptr && std::strcmp(e, "1") == 0;
}

// the attention kernels' function attributes: shared memory, and clusters of
// up to 16 CTAs (beyond the portable 8) for the 128-row kernel, once per
// process
template <bool POLY>
cudaError_t attn_set_attributes_t() {
  static cudaError_t done = cudaErrorNotReady;
  if (done == cudaErrorNotReady) {
    done = cudaFuncSetAttribute(attn_tc_kernel<POLY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kAttnSmem);
    if (done == cudaSuccess)
      done = cudaFuncSetAttribute(attn_tc_kernel<POLY>,
                                  cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (done == cudaSuccess)
      done = cudaFuncSetAttribute(attn_tc2_kernel<POLY>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, kAttn2Smem);
  }
  return done;
}
cudaError_t attn_set_attributes() { return attn_set_attributes_t<false>(); }

template <bool POLY>
cudaError_t attention_bf16_t(const ModelDims& md, const AttnPlan& ap, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap* tmQ, const void* q,
                             void* o, float* opart, float2* ml, const int32_t* lens,
                             const uint8_t* done, const int* n_active, int* err,
                             cudaStream_t st) {
  if (cudaError_t e = attn_set_attributes_t<POLY>(); e != cudaSuccess) return e;
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
  p.cluster = ap.cluster;
  p.q_tma = tmQ != nullptr && ap.G > 0 && kRowsCta % ap.G == 0 ? 1 : 0;
  p.Lcap = md.Lcap;
  const CUtensorMap qmap = tmQ != nullptr ? *tmQ : tmK;   // unread without q_tma
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)md.Dh));
  if (ap.rows == 2 * kRowsCta) {
    // two row tiles per CTA: one split writes O, more write partials
    if (ap.cluster > 1) return cudaErrorInvalidValue;
    dim3 grid2(ap.nsplit, (ap.rtiles + 1) / 2, ap.B * md.Hkv);
    cudaError_t e = launch_pdl(attn_tc2_kernel<POLY>, grid2, dim3(kAttn2Threads), kAttn2Smem, st,
                               tmK, tmV, qmap, p);
    if (e != cudaSuccess || ap.nsplit == 1) return e;
    const int rows_per_block = 8;
    dim3 g2(ap.B * md.Hkv, (ap.R + rows_per_block - 1) / rows_per_block);
    return launch_pdl(attn_combine_kernel, g2, dim3(32 * rows_per_block), 0, st,
                      (const float*)opart, (const float2*)ml, (__nv_bfloat16*)o, lens, done,
                      n_active, md.H, md.Hkv, ap.G, ap.C, ap.R, ap.chunk, ap.nsplit);
  }
  if (ap.rows != kRowsCta) return cudaErrorInvalidValue;
  dim3 grid(ap.nsplit, ap.rtiles, ap.B * md.Hkv);
  if (ap.cluster > 1) {
    // the splits of a (row tile, plane) as one cluster: no partials, no combine kernel
    if (ap.cluster != ap.nsplit || ap.cluster > kMaxCluster) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = kAttnSmem;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)ap.cluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, attn_tc_kernel<POLY>, tmK, tmV, qmap, p);
  }
  cudaError_t e =
      launch_pdl(attn_tc_kernel<POLY>, grid, dim3(192), kAttnSmem, st, tmK, tmV, qmap, p);
  if (e != cudaSuccess || ap.nsplit == 1) return e;
  const int rows_per_block = 8;
  dim3 g2(ap.B * md.Hkv, (ap.R + rows_per_block - 1) / rows_per_block);
  return launch_pdl(attn_combine_kernel, g2, dim3(32 * rows_per_block), 0, st,
                    (const float*)opart, (const float2*)ml, (__nv_bfloat16*)o, lens, done,
                    n_active, md.H, md.Hkv, ap.G, ap.C, ap.R, ap.chunk, ap.nsplit);
}

cudaError_t attention_bf16(const ModelDims& md, const AttnPlan& ap, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const CUtensorMap* tmQ, const void* q, void* o,
                           float* opart, float2* ml, const int32_t* lens, const uint8_t* done,
                           const int* n_active, int* err, cudaStream_t st) {
  return attn_poly()
             ? attention_bf16_t<true>(md, ap, tmK, tmV, tmQ, q, o, opart, ml, lens, done,
                                      n_active, err, st)
             : attention_bf16_t<false>(md, ap, tmK, tmV, tmQ, q, o, opart, ml, lens, done,
                                       n_active, err, st);
}

int attn_cluster_capacity(int n) {
  // clusters of n attention CTAs (one SM each) that can be resident at once
  static int cap[kMaxCluster + 1];
  static bool init = false;
  if (!init) {
    for (int i = 0; i <= kMaxCluster; ++i) cap[i] = -1;
    init = true;
  }
  if (n < 2 || n > kMaxCluster) return 0;
  if (cap[n] >= 0) return cap[n];
  if (attn_set_attributes() != cudaSuccess) {
    cudaGetLastError();
    return cap[n] = 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n, 1, 1);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = kAttnSmem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)n;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int num = 0;
  if (cudaOccupancyMaxActiveClusters(&num, attn_tc_kernel<false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    num = 0;
  }
  return cap[n] = num;
}

cudaError_t attention_f32(const ModelDims& md, int B, int C, const float* q, const float* kcache,
                          const float* vcache, float* o, const int32_t* lens,
                          const uint8_t* done, const int* n_active, int* err,
                          cudaStream_t st) {
  const float scale = (float)(1.0 / sqrt((double)md.Dh));
  const int threads = 128;
  cudaError_t e;
  if (md.Dh == 64)
    e = launch_pdl(attn_f32_kernel<64>, dim3(B * md.H), dim3(threads), 0, st, md.H, md.Hkv, C,
                   md.Lcap, q, kcache, vcache, o, lens, done, n_active, scale, err);
  else if (md.Dh == 128)
    e = launch_pdl(attn_f32_kernel<128>, dim3(B * md.H), dim3(threads), 0, st, md.H, md.Hkv, C,
                   md.Lcap, q, kcache, vcache, o, lens, done, n_active, scale, err);
  else if (md.Dh == 32)
    e = launch_pdl(attn_f32_kernel<32>, dim3(B * md.H), dim3(threads), 0, st, md.H, md.Hkv, C,
                   md.Lcap, q, kcache, vcache, o, lens, done, n_active, scale, err);
  else
    return cudaErrorInvalidValue;
  return e;
}

}  // namespace dlm
