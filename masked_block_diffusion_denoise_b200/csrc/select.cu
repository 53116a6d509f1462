// Selection half of the step, one CTA per canvas (kernel (c)):
//   1. combines the LM head's partials of each row (one per LM-head CTA)
//      into the candidate token, its confidence and the entropy;
//   2. ranks the uncommitted positions (bitonic sort in shared memory),
//      applies the threshold + quota rule or the entropy bound, forces
//      completion on the last step of the budget, handles EOS, re-noises the
//      rest and advances step / done.
// The selection follows the DiffusionGemma page (BlockRefinementScheduler,
// EntropyBoundScheduler), the course "Diffusion LLMs" section 12 (confidence
// order, ties to the lower position) and the Nemotron guide, section 6 (the
// last step fills every remaining mask).
#include <algorithm>

#include <cooperative_groups.h>

#include "kernels.h"

namespace dlm {

DLM_TRACE_STORAGE(sel)

namespace {

// combine the n_part partials of one row (a warp) into cand / conf / entropy:
//   M = max_j m_j,  S = sum_j s_j e^{m_j - M},  T = sum_j e^{m_j - M} (t_j + s_j (m_j - M)),
//   winner = the partial with the largest g (lowest index on ties).
// The partials are taken in chunks of 32 * kU: a chunk's maximum is a warp
// maximum, after which every lane's terms are independent of one another (no
// chain of pairwise merges); the lane sums and the winner meet in fixed
// butterflies, so the result does not depend on timing.
__device__ void reduce_row(const float* __restrict__ pr, int n_part, int lane, int32_t* cand,
                           float* conf, float* ent, int32_t* cand_sm, float* conf_sm,
                           float* ent_sm) {
  constexpr int kU = 5;   // one chunk covers one partial per SM of a 148-SM part
  float M = -CUDART_INF_F, s_l = 0.f, t_l = 0.f;
  float g_b = -CUDART_INF_F, zw_b = -CUDART_INF_F;
  int idx_b = 0x7fffffff;
  for (int j0 = 0; j0 < n_part; j0 += 32 * kU) {
    LmPart q[kU];
    bool ok[kU];
    float mloc = -CUDART_INF_F;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int j = j0 + lane + 32 * u;
      ok[u] = j < n_part;
      if (ok[u]) {
        // field-major row: each field of 32 partials is one 128-byte line
        q[u].m = pr[j];
        q[u].s = pr[n_part + j];
        q[u].t = pr[2 * n_part + j];
        q[u].g = pr[3 * n_part + j];
        q[u].zw = pr[4 * n_part + j];
        q[u].idx = __float_as_int(pr[5 * n_part + j]);
        ok[u] = q[u].m != -CUDART_INF_F;   // a tile with every column excluded
      }
      if (ok[u]) mloc = fmaxf(mloc, q[u].m);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, off));
    const float Mn = fmaxf(M, mloc);
    if (Mn == -CUDART_INF_F) continue;   // warp-uniform
    if (M != -CUDART_INF_F && Mn > M) {
      const float a = __expf(M - Mn);
      t_l = (t_l + s_l * (M - Mn)) * a;
      s_l *= a;
    }
    M = Mn;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (ok[u]) {
        const float d = q[u].m - M;
        const float w = __expf(d);
        s_l = fmaf(q[u].s, w, s_l);
        t_l = fmaf(w, fmaf(q[u].s, d, q[u].t), t_l);
        const bool better = q[u].g > g_b || (q[u].g == g_b && q[u].idx < idx_b);
        g_b = better ? q[u].g : g_b;
        zw_b = better ? q[u].zw : zw_b;
        idx_b = better ? q[u].idx : idx_b;
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    s_l += __shfl_xor_sync(0xffffffffu, s_l, off);
    t_l += __shfl_xor_sync(0xffffffffu, t_l, off);
    const float g_o = __shfl_xor_sync(0xffffffffu, g_b, off);
    const float zw_o = __shfl_xor_sync(0xffffffffu, zw_b, off);
    const int idx_o = __shfl_xor_sync(0xffffffffu, idx_b, off);
    const bool take = g_o > g_b || (g_o == g_b && idx_o < idx_b);
    g_b = take ? g_o : g_b;
    zw_b = take ? zw_o : zw_b;
    idx_b = take ? idx_o : idx_b;
  }
  if (lane == 0) {
    int32_t c = 0;
    float f = 0.f, h = 0.f;
    if (idx_b != 0x7fffffff && s_l > 0.f) {
      c = idx_b;
      f = expf(zw_b - M) / s_l;
      h = logf(s_l) - t_l / s_l;
    }
    *cand = c;
    *conf = f;
    *ent = h;
    *cand_sm = c;   // the block's own copy for the selection
    *conf_sm = f;
    *ent_sm = h;
  }
}

// float -> unsigned key with the same order (-0.0 folded onto +0.0)
__device__ __forceinline__ uint32_t ordered_bits(float x) {
  const uint32_t u = __float_as_uint(x + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kMaxC = 1024;
constexpr int kStageChunk = 32768;        // bytes per bulk copy of the partials
constexpr int kStageMax = 160 * 1024;     // partials staged up to this size per canvas

// positions after the first committed EOS become EOS and committed; returns
// the EOS position (or -1) and, through *filled, how many were filled
__device__ int eos_fill(int32_t* tok, uint8_t* com, int C, int eos_id, int* e_s, int* filled) {
  const int i = threadIdx.x;
  if (eos_id < 0) {
    *filled = 0;
    return -1;
  }
  if (i == 0) *e_s = C;
  __syncthreads();
  if (i < C && com[i] && tok[i] == eos_id) atomicMin(e_s, i);
  __syncthreads();
  const int e = *e_s;
  const bool f = (i < C && i > e && !com[i]);
  if (f) {
    tok[i] = eos_id;
    com[i] = 1;
  }
  *filled = __syncthreads_count(f);
  return e < C ? e : -1;
}

// One canvas per CTA, or, when the partials are given and the canvas is
// longer than 32 positions, one canvas per thread-block cluster of kcl CTAs:
// CTA r of the cluster reduces rows [r * rows_per, (r + 1) * rows_per) and
// writes their candidates, confidences and entropies into the shared memory
// of the cluster's first CTA, which then selects for the whole canvas.
__global__ void __launch_bounds__(1024) commit_kernel(SelectArgs a, int32_t* __restrict__ tokens,
                              uint8_t* __restrict__ committed, int32_t* __restrict__ step,
                              uint8_t* __restrict__ done, int32_t* __restrict__ eos_pos,
                              int32_t* __restrict__ prev_cand, int32_t* __restrict__ stable,
                              const float* __restrict__ part, int n_part, int stage_bytes,
                              int32_t* __restrict__ cand, float* __restrict__ conf,
                              float* __restrict__ ent, dlm_canvas_stats* stats,
                              const int* n_active, int* err, int kcl, int rows_per) {
  // timeline marks: 2 wait returned, 3 rows reduced, 4 keys sorted, 5 done
  DLM_TRACE_CTA(TRACE_COMMIT);
  // Inside a step (partials given) the direct predecessor is the LM head,
  // which writes only the partials: the active count and the canvas state
  // come from earlier kernels, complete once this kernel may start (every
  // kernel of the chain lets its successor launch only after its own wait),
  // and are read before the wait, through L2.  Given candidates (a call on
  // its own) the predecessor is unknown and everything is read after it.
  const bool early = part != nullptr;
  // stage_bytes > 0: this canvas's partials ([C][kLmFields][n_part] floats)
  // come into shared memory by bulk copies, a few instructions instead of
  // one load per field, partial and row from one SM
  extern __shared__ __align__(128) uint8_t stage_raw[];
  __shared__ uint64_t stage_bar;
  const bool staged = part != nullptr && stage_bytes > 0;
  if (staged) {
    if (threadIdx.x == 0) {
      mbar_init(&stage_bar, 1);
      fence_mbar_init();
    }
    __syncthreads();
  }
  if (!early) pdl_wait_then_release();
  const int rank = kcl > 1 ? (int)cooperative_groups::this_cluster().block_rank() : 0;
  const int b = blockIdx.x / kcl;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int i = threadIdx.x;
  const int C = a.C;
  const size_t base = (size_t)b * C;
  const int r0 = rank * rows_per, r1 = min(C, r0 + rows_per);   // this CTA's rows
  // the active count, this canvas's flag and state in one round trip; the
  // state goes to registers and reaches shared memory after the reduction
  const int na = n_active != nullptr ? __ldcg(n_active) : 1;
  const uint8_t dn = __ldcg(done + b);
  const int s = __ldcg(step + b);
  int32_t tok_r = 0;
  uint8_t com_r = 0;
  if (rank == 0 && i < C) {
    tok_r = __ldcg(tokens + base + i);
    com_r = __ldcg(committed + base + i);
  }
  // adaptive stopping's state and the counters, updated at the end, are
  // read here too (kept in shared memory), so that no load is left for the
  // end of the kernel
  __shared__ int32_t prev_s[kMaxC];
  __shared__ int32_t stable_s;
  __shared__ dlm_canvas_stats st0;
  const bool stopping = a.stop_entropy > 0.f;
  if (rank == 0 && stopping && i < C) prev_s[i] = __ldcg(prev_cand + base + i);
  if (rank == 0 && i == 0) {
    if (stopping) stable_s = __ldcg(stable + b);
    if (stats != nullptr) {
      const int32_t* sp = reinterpret_cast<const int32_t*>(stats + b);
      st0.steps_used = __ldcg(sp + 0);
      st0.committed_by_sampler = __ldcg(sp + 1);
      st0.forced_at_budget = __ldcg(sp + 2);
      st0.eos_autofill = __ldcg(sp + 3);
      st0.frozen = __ldcg(sp + 4);
      st0.edited = __ldcg(sp + 5);
    }
  }
  if (early) pdl_wait_then_release();
  if (threadIdx.x == 0) DLM_TRACE_MARK(2);
  // uniform over a cluster: its CTAs share the canvas
  if (na == 0 || dn) return;
  // this CTA's slice of the partials (stage_bytes is the largest slice)
  const int slice_bytes = (r1 - r0) * kLmFields * n_part * (int)sizeof(float);
  if (staged && i == 0) {
    mbar_arrive_expect_tx(&stage_bar, (uint32_t)slice_bytes);
    const uint8_t* src =
        reinterpret_cast<const uint8_t*>(part + (base + r0) * kLmFields * (size_t)n_part);
    for (int off = 0; off < slice_bytes; off += kStageChunk)
      bulk_load_global(stage_raw + off, src + off, (uint32_t)min(kStageChunk, slice_bytes - off),
                       &stage_bar);
  }
  __shared__ unsigned long long keys[kMaxC];
  __shared__ int32_t tok[kMaxC];
  __shared__ uint8_t com[kMaxC];
  __shared__ int32_t cand_s[kMaxC];   // this canvas's candidates, confidences, entropies
  __shared__ float conf_s[kMaxC], ent_s[kMaxC];
  __shared__ int e_s, k_s, krule_s;
  int P = 32;               // keys sorted: the next power of two >= C
  while (P < C) P <<= 1;
  if (part != nullptr) {
    if (staged && !mbar_wait_bounded(&stage_bar, 0, nullptr)) {
      raise_error(err, DLM_ETIMEOUT);
      mbar_wait_bounded(&stage_bar, 0, nullptr);   // the copies land before the CTA exits
    }
    // a6: the cross-tile reduction of this CTA's rows, one warp per row; the
    // results go to the cluster's first CTA (this CTA without a cluster)
    int32_t* cand_l = cand_s;
    float *conf_l = conf_s, *ent_l = ent_s;
    if (kcl > 1) {
      cooperative_groups::cluster_group cl = cooperative_groups::this_cluster();
      cand_l = cl.map_shared_rank(cand_s, 0);
      conf_l = cl.map_shared_rank(conf_s, 0);
      ent_l = cl.map_shared_rank(ent_s, 0);
    }
    for (int r = r0 + warp; r < r1; r += nw) {
      const size_t row = base + r;
      const float* pr = staged
                            ? reinterpret_cast<const float*>(stage_raw) + (r - r0) * kLmFields * n_part
                            : part + row * kLmFields * (size_t)n_part;
      reduce_row(pr, n_part, lane, cand + row, conf + row, ent + row, cand_l + r, conf_l + r,
                 ent_l + r);
    }
    if (kcl > 1) {
      // every row of the canvas is in the first CTA's shared memory
      cooperative_groups::this_cluster().sync();
      if (rank != 0) return;
    }
  } else if (i < C) {
    cand_s[i] = cand[base + i];
    conf_s[i] = conf[base + i];
    ent_s[i] = ent[base + i];
  }
  if (i < C) {
    tok[i] = tok_r;
    com[i] = com_r;
  }
  __syncthreads();
  if (i == 0) DLM_TRACE_MARK(3);

  int fill0 = 0, fill1 = 0;
  const int e0 = eos_fill(tok, com, C, a.eos_id, &e_s, &fill0);

  int nedit = 0;
  if (a.editing) {
    // token editing: a position committed before this step and before the
    // first committed EOS takes its candidate when that differs from the
    // token with confidence >= edit_thr (float32, -0 folded onto +0)
    const int lim = e0 < 0 ? C : e0;
    bool ed = false;
    if (i < lim && com[i]) {
      int c = cand_s[i];
      if (c != tok[i] && conf_s[i] + 0.0f >= a.edit_thr) {
        if (c < 0 || c >= a.V) {
          raise_error(err, DLM_EBOUNDS);
          c = 0;
        }
        tok[i] = c;
        ed = true;
      }
    }
    nedit = __syncthreads_count(ed);
  }

  if (stopping) {
    // adaptive stopping: the argmax of every position unchanged since the
    // previous step counts one stable step; with enough stable steps and a
    // mean entropy (float32, summed in position order) below the bound the
    // canvas freezes: every open position commits its candidate
    __shared__ int freeze_s;
    const bool same = (i >= C) || (cand_s[i] == prev_s[i]);
    const int all_same = __syncthreads_and(same);
    if (i < C) prev_cand[base + i] = cand_s[i];
    if (i == 0) {
      float total = 0.f;
      for (int j = 0; j < C; ++j) total = __fadd_rn(total, ent_s[j] + 0.0f);
      const float mean = __fdiv_rn(total, (float)C);
      const int st = all_same ? stable_s + 1 : 0;
      stable[b] = st;
      freeze_s = (st >= a.stability_steps && mean < a.stop_entropy) ? 1 : 0;
    }
    __syncthreads();
    if (freeze_s) {
      const bool opened = i < C && !com[i];
      if (opened) {
        int c = cand_s[i];
        if (c < 0 || c >= a.V) {
          raise_error(err, DLM_EBOUNDS);
          c = 0;
        }
        tok[i] = c;
        com[i] = 1;
      }
      const int nfrozen = __syncthreads_count(opened);
      const int e = eos_fill(tok, com, C, a.eos_id, &e_s, &fill1);
      if (i < C) {
        tokens[base + i] = tok[i];
        committed[base + i] = com[i];
      }
      const int all = __syncthreads_and(i >= C || com[i]);
      if (i == 0) {
        done[b] = all ? 1 : 0;
        step[b] = s + 1;
        eos_pos[b] = e;
        if (stats != nullptr) {
          dlm_canvas_stats& so = stats[b];
          so.steps_used = st0.steps_used + 1;
          so.frozen = st0.frozen + nfrozen;
          so.eos_autofill = st0.eos_autofill + fill0 + fill1;
          so.edited = st0.edited + nedit;
        }
      }
      return;
    }
  }

  const bool open = (i < C) && !com[i];
  unsigned long long key = ~0ull;
  if (open) {
    const uint32_t hi = a.eb ? ordered_bits(ent_s[i]) : ~ordered_bits(conf_s[i]);
    key = ((unsigned long long)hi << 32) | (unsigned)i;
  }
  if (i < P) keys[i] = key;
  const int nU = __syncthreads_count(open);
  const int nthr = __syncthreads_count(open && !a.eb && conf_s[i] >= a.threshold);

  if (P == 32) {
    // up to 32 keys: a bitonic network inside warp 0, in registers (the keys
    // are unique -- position in the low word -- so any sorting network gives
    // the same order)
    if (i < 32) {
      unsigned long long x = keys[i];
      for (int k = 2; k <= 32; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
          const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, j);
          const bool up = (i & k) == 0;
          const bool low = (i & j) == 0;
          x = (low == up) ? (x < y ? x : y) : (x < y ? y : x);
        }
      }
      keys[i] = x;
    }
    __syncthreads();
  } else {
    for (int k = 2; k <= P; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        const int ixj = i ^ j;
        if (i < P && ixj > i) {
          const unsigned long long x = keys[i], y = keys[ixj];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            keys[i] = y;
            keys[ixj] = x;
          }
        }
        __syncthreads();
      }
    }
  }

  if (i == 0) {
    DLM_TRACE_MARK(4);
    int k;
    if (a.eb) {
      k = 0;
      float run = 0.f;
      for (int j = 0; j < nU; ++j) {
        const int pos = (int)(keys[j] & 0xffffffffu);
        run = __fadd_rn(run, ent_s[pos] + 0.0f);
        if (run <= a.bound)
          ++k;
        else
          break;
      }
      if (nU > 0 && k < 1) k = 1;
    } else {
      k = nthr > a.quota ? nthr : a.quota;
      if (k > nU) k = nU;
    }
    krule_s = k;
    if (s >= a.S - 1) k = nU;
    k_s = k;
  }
  __syncthreads();
  const int k = k_s;
  if (i < k) {
    const int pos = (int)(keys[i] & 0xffffffffu);
    int c = cand_s[pos];
    if (c < 0 || c >= a.V) {
      raise_error(err, DLM_EBOUNDS);
      c = 0;
    }
    tok[pos] = c;
    com[pos] = 1;
  }
  __syncthreads();

  const int e = eos_fill(tok, com, C, a.eos_id, &e_s, &fill1);

  if (a.uniform && i < C && !com[i]) {
    const U32x4 w =
        philox10(U32x4{(uint32_t)b, (uint32_t)(s + 1), (uint32_t)i, kRenoiseWord}, a.seed_lo,
                 a.seed_hi);
    tok[i] = uniform_id(w.a, a.V);
  }
  if (i < C) {
    tokens[base + i] = tok[i];
    committed[base + i] = com[i];
  }
  const int all = __syncthreads_and(i >= C || com[i]);
  if (i == 0) {
    DLM_TRACE_MARK(5);
    done[b] = all ? 1 : 0;
    step[b] = s + 1;
    eos_pos[b] = e;
    if (stats != nullptr) {
      dlm_canvas_stats& so = stats[b];
      so.steps_used = st0.steps_used + 1;
      so.committed_by_sampler = st0.committed_by_sampler + k;
      so.forced_at_budget = st0.forced_at_budget + k - krule_s;
      so.eos_autofill = st0.eos_autofill + fill0 + fill1;
      so.edited = st0.edited + nedit;
    }
  }
}

}  // namespace

cudaError_t commit_step(const SelectArgs& a, int32_t* tokens, uint8_t* committed, int32_t* step,
                        uint8_t* done, int32_t* eos_pos, int32_t* prev_cand, int32_t* stable,
                        const float* part, int n_part, int32_t* cand, float* conf, float* ent,
                        dlm_canvas_stats* stats, const int* n_active, int* err, cudaStream_t st) {
  int P = 32;
  while (P < a.C) P <<= 1;
  if (P > kMaxC) return cudaErrorInvalidValue;
  if (part != nullptr) P = 1024;   // 32 warps for the row reductions
  // with partials, a canvas of more than 32 positions is reduced by a
  // cluster of up to 8 CTAs (an even number of rows each)
  int kcl = 1, rows_per = a.C;
  if (part != nullptr && a.C > 32) {
    kcl = std::min(8, (a.C + 31) / 32);
    rows_per = (a.C + kcl - 1) / kcl;
    rows_per += rows_per & 1;
    kcl = (a.C + rows_per - 1) / rows_per;
  }
  // a slice's partials go through shared memory when the largest fits and
  // every slice starts on a 16-byte boundary
  int stage_bytes = 0;
  if (part != nullptr) {
    const long long row_bytes = (long long)kLmFields * n_part * (long long)sizeof(float);
    const long long bytes = rows_per * row_bytes;
    if (bytes <= kStageMax && bytes % 16 == 0 && (a.C * row_bytes) % 16 == 0)
      stage_bytes = (int)bytes;
  }
  static cudaError_t attr = cudaErrorNotReady;   // per process; one device per process
  if (attr == cudaErrorNotReady)
    attr = cudaFuncSetAttribute(commit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kStageMax);
  if (attr != cudaSuccess) return attr;
  if (kcl == 1)
    return launch_pdl(commit_kernel, dim3(a.B), dim3(P), (size_t)stage_bytes, st, a, tokens,
                      committed, step, done, eos_pos, prev_cand, stable, part, n_part,
                      stage_bytes, cand, conf, ent, stats, n_active, err, 1, rows_per);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * kcl);
  cfg.blockDim = dim3(P);
  cfg.dynamicSmemBytes = (size_t)stage_bytes;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)kcl;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, commit_kernel, a, tokens, committed, step, done, eos_pos,
                            prev_cand, stable, part, n_part, stage_bytes, cand, conf, ent, stats,
                            n_active, err, kcl, rows_per);
}

}  // namespace dlm
