// tcgen05 GEMM engine for sm_100a: D[M][N] = A[M][K] . B[N][K]^T, bf16
// operands (both K-major, row-major in HBM), f32 accumulators in tensor
// memory.
//
// One persistent CTA per SM, three roles:
//   warp 0      TMA producer: streams 128x64 A and BNx64 B tiles (128-byte
//               swizzle) into a STAGES-deep shared-memory ring;
//   warp 1      MMA issuer: one thread issues tcgen05.mma 128xBNx16 into one
//               of two TMEM accumulators and frees ring slots with
//               tcgen05.commit;
//   warps 2..9  epilogue: tcgen05.ld the accumulator (one TMEM lane = one
//               output row per thread; two warpgroups, one column half each)
//               while the MMA warp fills the other accumulator.
// Epilogues:
//   EPI_F32  store f32 partial sums [split][M][N] (projections, split-K;
//            full logits for inspection).  Work units (m tile, n tile,
//            k split), m fastest, strided over the grid, so that CTAs that
//            run at the same time share the same B (weight) slab through L2.
//   EPI_QKV  (BN 256, K not split) the QKV projection: RoPE on q and k,
//            bf16 stores of q and of the canvas K / V into their cache slots.
//   EPI_RESID (BN 256, K not split) the output projection plus residual.
//   EPI_LM   the LM head's fused vocabulary reduction.  CTA c keeps m tile
//            c % m_tiles and walks vocabulary tiles c / m_tiles + k * slots;
//            each epilogue thread folds every tile of its row into one row
//            state and writes one partial per (row, CTA); logits never leave
//            the SM.  CTAs with the same slot read the same weight slab at
//            about the same time (L2 reuse across m tiles).
#include <cstdio>

#include "kernels.h"
#include "lm_epilogue.cuh"

namespace dlm {

DLM_TRACE_STORAGE(gemm)

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;   // one 128-byte swizzle atom of bf16 per row

// Shared memory: a ring of `stages` stages, each [B tile: BN rows x 128 B]
// [A tile: a_rows x 128 B], then a pad, the barriers and the row-state
// exchange.  With one M tile the A box holds only the rows in use (rounded up
// to 8); the MMA still reads 128 A rows, and rows past a_rows -- whatever
// follows in shared memory -- feed only accumulator rows the epilogue never
// reads.  The pad of (128 - a_rows) x 128 bytes keeps those reads of the last
// stage inside the allocation.  Smaller A tiles leave room for more stages
// of weights in flight.
template <int BN>
struct TcCfg {
  static constexpr int kMaxStages = 16;
  static constexpr int kBBytes = BN * 128;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kBarBytes = 512;       // mbarriers, TMEM slot, abort flag
  static constexpr int kXchBytes = 128 * 32;  // row states of the EPI_LM hand-over
  static constexpr int kSmem = 232448;        // the opt-in maximum per block
};

// sf: bytes of block scale factors per stage (NVFP4: 2 KB for the A rows'
// 128-row block, 2 KB per 128 B rows), after the A tile
__host__ __device__ constexpr int tc_stage_bytes(int BN, int a_rows, int sf = 0) {
  return (BN + a_rows) * 128 + sf;
}
__host__ __device__ constexpr int tc_bar_offset(int BN, int a_rows, int stages, int sf = 0) {
  return stages * tc_stage_bytes(BN, a_rows, sf) + (128 - a_rows) * 128;
}
template <int BN>
constexpr int tc_stages(int a_rows, int sf = 0) {
  using Cfg = TcCfg<BN>;
  const int room = Cfg::kSmem - 1024 - Cfg::kBarBytes - Cfg::kXchBytes - (128 - a_rows) * 128;
  const int n = room / tc_stage_bytes(BN, a_rows, sf);
  return n < Cfg::kMaxStages ? n : Cfg::kMaxStages;
}
__host__ __device__ constexpr int tc_sf_bytes(int BN, bool f4) { return f4 ? 2048 * (1 + BN / 128) : 0; }

struct TcParams {
  int M, N, K;
  int m_tiles, n_tiles, splits, units, kblocks;
  int a_rows, stages;    // A box rows (multiple of 8, <= 128), ring stages
  float* out;
  float* part;           // EPI_LM partials, [M][kLmFields][slots]
  LmEpi epi;
  ProjEpi proj;
  const uint8_t* done;   // [B] canvases that are finished (LM rows skipped)
  const int* n_active;   // whole launch skipped when *n_active == 0
  int* err;
  int trace_kind;        // device timeline (DLM_TRACE builds), -1: not traced
  // failure-detection test: the producer issues no loads, so the MMA warp's
  // waits for them run out after wait_ns and the launch records DLM_ETIMEOUT
  int withhold_loads;
  uint64_t wait_ns;      // limit of the MMA warp's waits for ring stages
  // NVFP4 operands: block scale factors of A and B in the block-scaled MMA's
  // layout, [row block of 128][k group of 64][512 bytes]; kg = K / 64
  const uint8_t* sfa;
  const uint8_t* sfb;
  int kg;
};

__device__ __forceinline__ void unit_coords(const TcParams& p, int u, int& m, int& n, int& kb0,
                                            int& kb1) {
  m = u % p.m_tiles;
  const int rest = u / p.m_tiles;
  n = rest % p.n_tiles;
  const int split = rest / p.n_tiles;
  kb0 = (int)(((long long)split * p.kblocks) / p.splits);
  kb1 = (int)(((long long)(split + 1) * p.kblocks) / p.splits);
}

// The k-th unit of this CTA.  EPI_F32: units strided over the grid.  EPI_LM:
// the CTA keeps one m tile and walks the vocabulary tiles slot, slot+slots, ...
// (slots = gridDim.x / m_tiles), so the epilogue can fold all of them into
// one row state and write a single partial per (row, CTA).
template <int EPI>
__device__ __forceinline__ bool get_unit(const TcParams& p, int k, int& m, int& n, int& kb0,
                                         int& kb1, int& split) {
  if constexpr (EPI == EPI_LM) {
    const int slots = gridDim.x / p.m_tiles;
    m = blockIdx.x % p.m_tiles;
    n = blockIdx.x / p.m_tiles + k * slots;
    kb0 = 0;
    kb1 = p.kblocks;
    split = 0;
    return n < p.n_tiles;
  } else {
    const int u = blockIdx.x + k * gridDim.x;
    if (u >= p.units) return false;
    unit_coords(p, u, m, n, kb0, kb1);
    split = (u / p.m_tiles) / p.n_tiles;
    return true;
  }
}

constexpr int kGemmThreads = 320;   // producer, MMA, 8 epilogue warps

// Scale 32 accumulator columns of one row to logits: v_j * (a * s_j), the
// factor rounded to float32 first (e4m3 operands with per-row scales).
__device__ __forceinline__ void scale_chunk(float (&v)[32], float a, const float* __restrict__ cs) {
  const float4* c4 = reinterpret_cast<const float4*>(cs);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 sc = c4[j];
    v[4 * j + 0] = __fmul_rn(v[4 * j + 0], __fmul_rn(a, sc.x));
    v[4 * j + 1] = __fmul_rn(v[4 * j + 1], __fmul_rn(a, sc.y));
    v[4 * j + 2] = __fmul_rn(v[4 * j + 2], __fmul_rn(a, sc.z));
    v[4 * j + 3] = __fmul_rn(v[4 * j + 3], __fmul_rn(a, sc.w));
  }
}

// F8: e4m3 operands (kind::f8f6f4); a k-block is then 128 elements, the same
// 128 bytes per row as 64 bf16 elements, so ring, swizzle and descriptors
// are shared.  F4: NVFP4 operands (kind::mxf4nvf4, packed e2m1, 256
// elements per 128-byte row of a k-block) with e4m3 scale factors per 16
// elements: each stage also carries the k-block's scale factors of the A and
// B rows (2 KB per 128-row block), which the MMA thread copies into tensor
// memory right before the stage's four MMAs (tcgen05 operations of one
// thread run in order, so one scale-factor area serves every stage).
template <int BN, int EPI, bool F8, bool F4 = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const TcParams p) {
  using Cfg = TcCfg<BN>;
  static_assert(!(F4 && (F8 || BN != 128)), "NVFP4 tiles are 128 wide");
  constexpr int kBKe = F4 ? 4 * kBK : (F8 ? 2 * kBK : kBK);   // elements per k-block
  constexpr int kSf = tc_sf_bytes(BN, F4);
  constexpr uint32_t kTmemAlloc = F4 ? 512 : Cfg::kTmemCols;   // + scale-factor columns
  constexpr uint32_t kSfaCol = 2 * BN, kSfbCol = 2 * BN + 16;
  constexpr int kBX = F4 ? 2 * kBK : kBKe;   // TMA x coordinate (bytes for 8/4-bit) per k-block
  // timeline marks: 2 wait returned, 3 / 4 first / last ring stage full,
  // 5 first accumulator ready, 6 last tile's epilogue done
  DLM_TRACE_CTA(p.trace_kind);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  const int stage_bytes = tc_stage_bytes(BN, p.a_rows, kSf);
  const uint32_t a_bytes = (uint32_t)p.a_rows * 128u;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + tc_bar_offset(BN, p.a_rows, stages, kSf));
  uint64_t* empty = full + Cfg::kMaxStages;
  uint64_t* tfull = empty + Cfg::kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemAlloc);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The weights (B) do not depend on the previous kernel: before waiting for
  // it, the producer puts the B tiles of the first ring stages in flight
  // (expected bytes raised, no arrival yet).  Right after the wait, before
  // anything else, it issues those stages' A tiles; the active count is read
  // only then, so its round trip overlaps the A loads.  Weights are read once
  // per launch: they stream through L2 with evict_first.
  int pre = 0;
  uint64_t pol_stream = 0;
  int m_first = 0, kb_first = 0;
  if (warp == 0 && lane == 0) {
    pol_stream = l2_evict_first_policy();
    int n0, kb1, sp0;
    if (!p.withhold_loads && get_unit<EPI>(p, 0, m_first, n0, kb_first, kb1, sp0)) {
      pre = min(stages, kb1 - kb_first);
      for (int s = 0; s < pre; ++s) {
        const int kb = kb_first + s;
        mbar_expect_tx(&full[s], Cfg::kBBytes + (F4 ? 2048u * (BN / 128) : 0u));
        tma_load_2d_hint(smem + s * stage_bytes, &tmB, &full[s], kb * kBX, n0 * BN, pol_stream);
        if constexpr (F4) {
          uint8_t* sfb_s = smem + s * stage_bytes + Cfg::kBBytes + a_bytes + 2048;
          for (int rb = 0; rb < BN / 128; ++rb)
            bulk_load_global(sfb_s + rb * 2048,
                             p.sfb + ((size_t)(n0 * (BN / 128) + rb) * p.kg + 4 * kb) * 512, 2048,
                             &full[s]);
        }
      }
    }
  }
  // the prologue above touched only shared and tensor memory and weights
  pdl_wait_then_release();
  if (warp == 0 && lane == 0) {
    DLM_TRACE_MARK(2);
    // the A tiles of the stages whose B tiles are in flight (the A buffer is
    // always allocated, so these loads are issued even when the step turns
    // out to have nothing to do)
    for (int s = 0; s < pre; ++s) {
      mbar_arrive_expect_tx(&full[s], a_bytes + (F4 ? 2048u : 0u));
      tma_load_2d(smem + s * stage_bytes + Cfg::kBBytes, &tmA, &full[s], (kb_first + s) * kBX,
                  m_first * kBM);
      if constexpr (F4)
        bulk_load_global(smem + s * stage_bytes + Cfg::kBBytes + a_bytes,
                         p.sfa + ((size_t)m_first * p.kg + 4 * (kb_first + s)) * 512, 2048,
                         &full[s]);
    }
  }
  const bool skip = p.n_active != nullptr && *p.n_active == 0;

  if (skip) {
    // nothing to do this step: land the early tiles, then teardown
    if (warp == 0 && lane == 0)
      for (int s = 0; s < pre; ++s) mbar_wait_bounded(&full[s], 0u, nullptr);
  } else if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && !p.withhold_loads) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      int m, n, kb0, kb1, split;
      for (int it = 0; ok && get_unit<EPI>(p, it, m, n, kb0, kb1, split); ++it) {
        for (int kb = kb0; kb < kb1; ++kb) {
          // The first `pre` stages (their first use of the ring) are already
          // in flight.  Their empty slots are not waited for: the MMA may have
          // consumed and released them already, and a wait on the released
          // phase would then wait for the next one.
          if (issued >= pre) {
            if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t* sb = smem + stage * stage_bytes;
            uint8_t* sa = sb + Cfg::kBBytes;
            mbar_arrive_expect_tx(&full[stage], (uint32_t)stage_bytes);
            tma_load_2d(sa, &tmA, &full[stage], kb * kBX, m * kBM);
            tma_load_2d_hint(sb, &tmB, &full[stage], kb * kBX, n * BN, pol_stream);
            if constexpr (F4) {
              uint8_t* sfa_s = sa + a_bytes;
              bulk_load_global(sfa_s, p.sfa + ((size_t)m * p.kg + 4 * kb) * 512, 2048,
                               &full[stage]);
              for (int rb = 0; rb < BN / 128; ++rb)
                bulk_load_global(sfa_s + 2048 + rb * 2048,
                                 p.sfb + ((size_t)(n * (BN / 128) + rb) * p.kg + 4 * kb) * 512,
                                 2048, &full[stage]);
            }
          }
          ++issued;
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let the copies already in flight land before the CTA exits
        if (issued < pre) {
          for (int s = 0; s < pre; ++s) mbar_wait_bounded(&full[s], 0u, nullptr);
        } else {
          int st = stage, ph = phase;
          for (int i = 0; i < stages && i < issued; ++i) {
            if (--st < 0) {
              st = stages - 1;
              ph ^= 1;
            }
            mbar_wait_bounded(&full[st], (uint32_t)ph, nullptr);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = F4 ? idesc_nvfp4_f32(kBM, BN)
                                    : (F8 ? idesc_e4m3_f32(kBM, BN) : idesc_bf16_f32(kBM, BN));
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      int m, n, kb0, kb1, split;
      for (int it = 0; ok && get_unit<EPI>(p, it, m, n, kb0, kb1, split); ++it) {
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          if (it == 0 && kb == kb0) DLM_TRACE_MARK(3);
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + stage * stage_bytes);
          const uint32_t sa = sb + Cfg::kBBytes;
          if constexpr (F4) {
            // the k-block's scale factors into tensor memory: per MMA (64
            // elements) 4 columns of A's and BN/32 columns of B's
            const uint32_t sfa_s = sa + a_bytes, sfb_s = sfa_s + 2048;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              tmem_cp_32x128b_x4(tmem_base + kSfaCol + 4 * k, rows16_desc(sfa_s + k * 512));
#pragma unroll
              for (int rb = 0; rb < BN / 128; ++rb)
                tmem_cp_32x128b_x4(tmem_base + kSfbCol + (BN / 32) * k + 4 * rb,
                                   rows16_desc(sfb_s + rb * 2048 + k * 512));
            }
          }
          // four instructions of 32 bytes of K per 128-byte k-block
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if constexpr (F4)
              umma_nvfp4(d_tmem, sw128_desc(sa + k * 32), sw128_desc(sb + k * 32), idesc,
                         tmem_base + kSfaCol + 4 * k, tmem_base + kSfbCol + (BN / 32) * k,
                         (kb > kb0 || k > 0) ? 1u : 0u);
            else if constexpr (F8)
              umma_e4m3(d_tmem, sw128_desc(sa + k * 32), sw128_desc(sb + k * 32), idesc,
                        (kb > kb0 || k > 0) ? 1u : 0u);
            else
              umma_bf16(d_tmem, sw128_desc(sa + k * 32), sw128_desc(sb + k * 32), idesc,
                        (kb > kb0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        DLM_TRACE_MARK(4);
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // every MMA issued has completed before TMEM is released
      umma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0, nullptr);
    }
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    // two warpgroups; warp w reads TMEM lanes 32*(w%4).. and warpgroup
    // (w-2)/4 takes one half of the columns of every accumulator tile
    const int quad = warp & 3;            // TMEM lanes 32*quad .. 32*quad+31
    const int wg = (warp - 2) >> 2;
    constexpr int kHalfN = BN / 2;
    const int cb = wg * kHalfN;           // first column of this warpgroup
    int acc = 0;
    uint32_t acc_phase = 0;
    int m = 0, n, kb0, kb1, split;
    // EPI_LM: one row state for all vocabulary tiles of this CTA
    RowState rs;
    rs_init(rs);
    int lm_row = -1, lm_canvas = 0, lm_pos = 0, lm_step = 0;
    bool lm_live = false;
    float lm_inv_t = 1.f;
    float lm_a = 0.f;   // F8: the row's scale
    if constexpr (EPI == EPI_LM) {
      m = blockIdx.x % p.m_tiles;
      lm_row = m * kBM + quad * 32 + lane;
      lm_canvas = lm_row / p.epi.C;
      lm_pos = lm_row - lm_canvas * p.epi.C;
      lm_live = lm_row < p.M && (p.done == nullptr || p.done[lm_canvas] == 0);
      lm_step = lm_live ? p.epi.step[lm_canvas] : 0;
      lm_inv_t = lm_inv_temp(p.epi, lm_step);
      if constexpr (F8 || F4) lm_a = lm_live ? p.epi.row_scale[lm_row] : 0.f;
    }
    for (int it = 0; get_unit<EPI>(p, it, m, n, kb0, kb1, split); ++it) {
      if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag)) break;
      if (it == 0 && warp == 2 && lane == 0) DLM_TRACE_MARK(5);
      tc_fence_after();
      const int row0 = m * kBM + quad * 32;
      const int row = row0 + lane;
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
      if (row0 < p.M) {   // warp-uniform: tcgen05.ld is a warp-wide instruction
        if constexpr (EPI == EPI_F32) {
          float* orow = p.out + ((size_t)split * p.M + row) * p.N;
#pragma unroll 1
          for (int c = cb; c < cb + kHalfN; c += 32) {
            float v[32];
            tmem_ld32(taddr + c, v);
            const int col0 = n * BN + c;
            if constexpr (F8 || F4) {
              if (p.epi.col_scale != nullptr)
                scale_chunk(v, row < p.M ? p.epi.row_scale[row] : 0.f, p.epi.col_scale + col0);
            }
            if (row < p.M) {
              if (col0 + 32 <= p.N) {
                float4* dst = reinterpret_cast<float4*>(orow + col0);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
              } else {
                for (int j = 0; j < 32; ++j)
                  if (col0 + j < p.N) orow[col0 + j] = v[j];
              }
            }
          }
        } else if constexpr (EPI == EPI_LM) {
#pragma unroll 1
          for (int c = cb; c < cb + kHalfN; c += 32) {
            float v[32];
            tmem_ld32(taddr + c, v);
            if constexpr (F8 || F4) scale_chunk(v, lm_a, p.epi.col_scale + n * BN + c);
            if (lm_live)
              rs_update<32>(rs, v, n * BN + c, lm_inv_t, p.epi, lm_canvas, lm_pos, lm_step);
          }
        } else if constexpr (EPI == EPI_QKV) {
          // 128-column heads, each as two units of 32 rotary pairs (j, j+64),
          // j in [32c, 32c+32): rotate q and k, store q rows and the canvas
          // K / V into the cache slots.  The BN/64 units of a tile are split
          // evenly between the two warpgroups.  The row's cache slot is read
          // once per tile, and each unit's cos/sin (16-byte loads) are in
          // flight while its accumulator columns come out of tensor memory.
          const ProjEpi& pe = p.proj;
          const int seq = row / pe.C, p_in = row - seq * pe.C;
          const bool live = row < p.M && (p.done == nullptr || p.done[seq] == 0);
          const int pos = live ? pe.lens[seq] + p_in : 0;
          const bool pos_ok = live && DLM_IN_BOUNDS(pos, pe.Lcap, p.err);
          constexpr int kUnits = BN / 128 * 2;
#pragma unroll 1
          for (int u = wg * kUnits / 2; u < (wg + 1) * kUnits / 2; ++u) {
            const int hc = u >> 1, c = u & 1;
            const int head = (n * BN) / 128 + hc;
            const bool store = pos_ok && head < pe.H + 2 * pe.Hkv;
            __nv_bfloat16* dst = nullptr;
            if (store) {
              if (head < pe.H) {
                dst = (__nv_bfloat16*)pe.q + ((size_t)row * pe.H + head) * 128;
              } else if (head < pe.H + pe.Hkv) {
                dst = (__nv_bfloat16*)pe.kcache +
                      (((size_t)seq * pe.Hkv + (head - pe.H)) * pe.Lcap + pos) * 128;
              } else {
                dst = (__nv_bfloat16*)pe.vcache +
                      (((size_t)seq * pe.Hkv + (head - pe.H - pe.Hkv)) * pe.Lcap + pos) * 128;
              }
            }
            const bool rotate = store && pe.rope != nullptr && head < pe.H + pe.Hkv;
            // two halves of 16 pairs
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
              const int j0 = c * 32 + h * 16;   // first pair of this half
              float4 cs[8];                     // cos/sin of its 16 pairs, two a load
              if (rotate) {
                const float4* src = reinterpret_cast<const float4*>(pe.rope + (size_t)pos * 64 + j0);
#pragma unroll
                for (int j = 0; j < 8; ++j) cs[j] = src[j];
              }
              uint32_t lo_raw[16], hi_raw[16];
              tmem_ld16_nowait(taddr + hc * 128 + j0, lo_raw);
              tmem_ld16_nowait(taddr + hc * 128 + 64 + j0, hi_raw);
              tmem_wait_ld();
              if (store) {
                float lo[16], hi[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  lo[j] = __uint_as_float(lo_raw[j]);
                  hi[j] = __uint_as_float(hi_raw[j]);
                }
                if (rotate) {
#pragma unroll
                  for (int j = 0; j < 16; ++j) {
                    const float2 r = (j & 1) ? make_float2(cs[j >> 1].z, cs[j >> 1].w)
                                             : make_float2(cs[j >> 1].x, cs[j >> 1].y);
                    const float a = lo[j], b2 = hi[j];
                    lo[j] = a * r.x - b2 * r.y;
                    hi[j] = b2 * r.x + a * r.y;
                  }
                }
#pragma unroll
                for (int q4 = 0; q4 < 2; ++q4) {
                  uint4 w, v;
                  w.x = pack_bf16(lo[8 * q4 + 0], lo[8 * q4 + 1]);
                  w.y = pack_bf16(lo[8 * q4 + 2], lo[8 * q4 + 3]);
                  w.z = pack_bf16(lo[8 * q4 + 4], lo[8 * q4 + 5]);
                  w.w = pack_bf16(lo[8 * q4 + 6], lo[8 * q4 + 7]);
                  v.x = pack_bf16(hi[8 * q4 + 0], hi[8 * q4 + 1]);
                  v.y = pack_bf16(hi[8 * q4 + 2], hi[8 * q4 + 3]);
                  v.z = pack_bf16(hi[8 * q4 + 4], hi[8 * q4 + 5]);
                  v.w = pack_bf16(hi[8 * q4 + 6], hi[8 * q4 + 7]);
                  reinterpret_cast<uint4*>(dst + j0)[q4] = w;
                  reinterpret_cast<uint4*>(dst + 64 + j0)[q4] = v;
                }
              }
            }
          }
        } else {
          // EPI_RESID: y = x + acc
          const ProjEpi& pe = p.proj;
          const int seq = row / pe.C;
          const bool live = row < p.M && (p.done == nullptr || p.done[seq] == 0);
#pragma unroll 1
          for (int c = cb; c < cb + kHalfN; c += 32) {
            float v[32];
            tmem_ld32(taddr + c, v);
            const int col0 = n * BN + c;
            if (live && col0 < p.N) {
              const uint4* xs =
                  reinterpret_cast<const uint4*>((const __nv_bfloat16*)pe.x + (size_t)row * p.N + col0);
              uint4* ys = reinterpret_cast<uint4*>((__nv_bfloat16*)pe.y + (size_t)row * p.N + col0);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const uint4 xv = xs[q4];
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                uint32_t yw[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const __nv_bfloat162 x2 = *reinterpret_cast<const __nv_bfloat162*>(&xw[u]);
                  const float2 xf = __bfloat1622float2(x2);
                  yw[u] = pack_bf16(xf.x + v[8 * q4 + 2 * u], xf.y + v[8 * q4 + 2 * u + 1]);
                }
                ys[q4] = make_uint4(yw[0], yw[1], yw[2], yw[3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (warp == 2 && lane == 0) DLM_TRACE_MARK(6);
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if constexpr (EPI == EPI_LM) {
      // the two warpgroups' states of a row: warpgroup 1 hands its state over
      // through shared memory, warpgroup 0 combines (fixed order) and stores
      RowState* xch = reinterpret_cast<RowState*>(reinterpret_cast<uint8_t*>(full) + Cfg::kBarBytes);
      const int lr = quad * 32 + lane;
      if (wg == 1) xch[lr] = rs;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (wg == 0) {
        const RowState both = rs_combine(rs, xch[lr]);
        const int slots = gridDim.x / p.m_tiles;
        if (lm_live) rs_store(p.part, slots, (size_t)lm_row, blockIdx.x / p.m_tiles, both);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemAlloc);
  }
  if (threadIdx.x == 0 && *abort_flag) raise_error(p.err, DLM_ETIMEOUT);
}

// EPI_LM: whole multiples of m_tiles CTAs (each keeps one m tile), at most
// one CTA per SM per m tile slot; EPI_F32: one CTA per SM or per unit.
int tc_grid(int units, int m_tiles, int n_tiles, int epi, int num_sms) {
  if (epi == EPI_LM) {
    int slots = num_sms / m_tiles;
    if (slots < 1) slots = 1;
    if (slots > n_tiles) slots = n_tiles;
    return slots * m_tiles;
  }
  return units < num_sms ? units : num_sms;
}

template <int BN, int EPI, bool F8 = false, bool F4 = false>
cudaError_t launch_tc(const CUtensorMap& tmA, const CUtensorMap& tmB, const TcParams& p,
                      int num_sms, cudaStream_t st) {
  using Cfg = TcCfg<BN>;
  static bool attr_set = false;   // per process; one device is used per process
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI, F8, F4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = tc_grid(p.units, p.m_tiles, p.n_tiles, EPI, num_sms);
  return launch_pdl(gemm_tc_kernel<BN, EPI, F8, F4>, dim3(grid), dim3(kGemmThreads), Cfg::kSmem,
                    st, tmA, tmB, p);
}

}  // namespace

cudaError_t gemm_tc(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmPlan& plan,
                    const GemmIO& io, int num_sms, cudaStream_t st) {
  TcParams p{};
  p.M = plan.M;
  p.N = plan.N;
  p.K = plan.K;
  p.m_tiles = (plan.M + kBM - 1) / kBM;
  p.n_tiles = (plan.N + plan.BN - 1) / plan.BN;
  p.splits = plan.splits;
  const int kbe = plan.f4 ? 4 * kBK : (plan.f8 ? 2 * kBK : kBK);   // elements per k-block
  p.kblocks = (plan.K + kbe - 1) / kbe;
  p.units = p.m_tiles * p.n_tiles * p.splits;
  p.a_rows = gemm_tc_a_rows(plan.M);
  const int sf = tc_sf_bytes(plan.BN, plan.f4 != 0);
  p.stages = plan.BN == 128 ? tc_stages<128>(p.a_rows, sf) : tc_stages<256>(p.a_rows, sf);
  p.out = io.out;
  p.part = io.part;
  p.epi = io.epi;
  p.epi.n_tiles = p.n_tiles;
  p.proj = io.proj;
  p.done = io.done;
  p.n_active = io.n_active;
  p.err = io.err;
  p.trace_kind = io.trace_kind;
  p.withhold_loads = io.withhold_loads;
  p.wait_ns = io.withhold_loads ? 20000000ull : kWaitLimitNs;   // 20 ms in the test
  p.sfa = io.sfa;
  p.sfb = io.sfb;
  p.kg = plan.K / 64;
  if (plan.f4) {
    // NVFP4 operands: the LM head and its full-logit inspection, 128-wide tiles
    if (plan.BN != 128 || plan.K % 256 != 0 || io.sfa == nullptr || io.sfb == nullptr)
      return cudaErrorInvalidValue;
    if (plan.epi == EPI_LM) return launch_tc<128, EPI_LM, false, true>(tmA, tmB, p, num_sms, st);
    if (plan.epi == EPI_F32) return launch_tc<128, EPI_F32, false, true>(tmA, tmB, p, num_sms, st);
    return cudaErrorInvalidValue;
  }
  if (plan.f8) {
    // e4m3 operands: the LM head and its full-logit inspection only
    if (plan.epi == EPI_LM)
      return plan.BN == 128 ? launch_tc<128, EPI_LM, true>(tmA, tmB, p, num_sms, st)
                            : launch_tc<256, EPI_LM, true>(tmA, tmB, p, num_sms, st);
    if (plan.epi == EPI_F32)
      return plan.BN == 128 ? launch_tc<128, EPI_F32, true>(tmA, tmB, p, num_sms, st)
                            : launch_tc<256, EPI_F32, true>(tmA, tmB, p, num_sms, st);
    return cudaErrorInvalidValue;
  }
  if (plan.BN == 128) {
    switch (plan.epi) {
      case EPI_LM: return launch_tc<128, EPI_LM>(tmA, tmB, p, num_sms, st);
      case EPI_QKV: return launch_tc<128, EPI_QKV>(tmA, tmB, p, num_sms, st);
      case EPI_RESID: return launch_tc<128, EPI_RESID>(tmA, tmB, p, num_sms, st);
      default: return launch_tc<128, EPI_F32>(tmA, tmB, p, num_sms, st);
    }
  }
  switch (plan.epi) {
    case EPI_LM: return launch_tc<256, EPI_LM>(tmA, tmB, p, num_sms, st);
    case EPI_QKV: return launch_tc<256, EPI_QKV>(tmA, tmB, p, num_sms, st);
    case EPI_RESID: return launch_tc<256, EPI_RESID>(tmA, tmB, p, num_sms, st);
    default: return launch_tc<256, EPI_F32>(tmA, tmB, p, num_sms, st);
  }
}

int gemm_tc_smem_bytes(int BN) { return BN == 128 ? TcCfg<128>::kSmem : TcCfg<256>::kSmem; }

int gemm_tc_a_rows(int M) { return M >= kBM ? kBM : ((M + 7) / 8) * 8; }

int gemm_tc_lm_partials(const GemmPlan& plan, int num_sms) {
  const int m_tiles = (plan.M + kBM - 1) / kBM;
  const int n_tiles = (plan.N + plan.BN - 1) / plan.BN;
  return tc_grid(m_tiles * n_tiles, m_tiles, n_tiles, EPI_LM, num_sms) / m_tiles;
}

}  // namespace dlm
