// Host side of the C ABI declared in include/dlm.h: context, argument
// validation, work plans, TMA tensor maps, the kernel sequence of one
// denoising step and the CUDA-graph replay of a block.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "kernels.h"

using namespace dlm;

namespace {

thread_local std::string g_create_error;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

struct GraphEntry {
  std::vector<uint8_t> key;
  cudaGraphExec_t exec = nullptr;
  int launches = 0;
};

}  // namespace

struct dlm_ctx {
  dlm_model_desc d{};
  ModelDims md{};
  int dev = 0, num_sms = 148;
  bool bf16 = true;
  // e4m3 LM head: quantised weights, their scales, the step's quantised rows
  bool lm_f8 = false;
  // NVFP4 LM head: as above with packed e2m1 elements and, in addition, the
  // e4m3 block scales of weights and rows in the block-scaled MMA's layout
  bool lm_f4 = false;
  uint8_t *w_lm_q = nullptr, *yq = nullptr;
  uint8_t *lm_sf = nullptr, *y_sf = nullptr;
  size_t lm_sf_bytes = 0, y_sf_bytes = 0;
  float *s_lm = nullptr, *s_y = nullptr;
  size_t s_lm_count = 0;
  size_t es = 2;
  const void *emb = nullptr, *w_o = nullptr, *w_lm = nullptr;
  void* w_qkv = nullptr;
  int Nqkv = 0;
  void *kc = nullptr, *vc = nullptr;
  int Lcap = 0;
  std::vector<int> lens_h;
  int32_t* lens_d = nullptr;
  int Mmax = 0;
  void *x = nullptr, *q = nullptr, *o = nullptr, *y = nullptr;
  float* part = nullptr;
  size_t part_floats = 0;
  float* opart = nullptr;
  size_t opart_floats = 0;
  float2* ml = nullptr;
  size_t ml_count = 0;
  float* lmpart = nullptr;   // LM-head partials, [M][kLmFields][n_part]
  int32_t* cand = nullptr;
  float *conf = nullptr, *ent = nullptr;
  float2* rope = nullptr;
  int* n_active = nullptr;
  int* err = nullptr;
  // device copies of a canvas for the host-buffer entry point
  int32_t *h_tok = nullptr, *h_step = nullptr, *h_eos = nullptr, *h_prev = nullptr,
          *h_stable = nullptr;
  uint8_t *h_com = nullptr, *h_done = nullptr;
  dlm_canvas_stats* h_stats = nullptr;
  std::map<std::tuple<const void*, uint64_t, uint64_t, uint32_t>, CUtensorMap> maps;
  CUtensorMap tmK{}, tmV{};
  CUtensorMap tmQ{};
  bool has_tmQ = false;   // the query tile by TMA (G divides 128)
  std::vector<GraphEntry> graphs;
  std::map<std::vector<int>, AttnPlan> plans;   // attention split plans
  cudaStream_t cap = nullptr;
  std::string msg;
  int launches = 0;
  int withhold_gemms = 0;   // failure-detection test: GEMM launches left to starve
  // measurement hook: events around one stage
  int ev_stage = -1;
  std::vector<cudaEvent_t> ev;
  int ev_step = 0;
  std::vector<void*> owned;
};

namespace {

int fail(dlm_ctx* c, int code, const std::string& what) {
  if (c) {
    if (c->msg.empty()) c->msg = what;
  } else {
    g_create_error = what;
  }
  return code;
}

int cuda_fail(dlm_ctx* c, const char* where, cudaError_t e) {
  return fail(c, DLM_ECUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

#define CK(call)                                            \
  do {                                                      \
    cudaError_t e_ = (call);                                \
    if (e_ != cudaSuccess) return cuda_fail(ctx, #call, e_); \
  } while (0)

template <typename T>
int dalloc(dlm_ctx* ctx, T** p, size_t bytes) {
  void* v = nullptr;
  cudaError_t e = cudaMalloc(&v, bytes < 256 ? 256 : bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(ctx, DLM_ENOMEM, "cudaMalloc of " + std::to_string(bytes) + " bytes failed");
  }
  ctx->owned.push_back(v);
  *p = reinterpret_cast<T*>(v);
  return DLM_OK;
}

// row-major [rows][cols] of bf16 (u8 = false) or one-byte e4m3 (u8 = true);
// the box is 128 bytes of a row (the 128-byte swizzle span) x box_rows
const CUtensorMap* map2d(dlm_ctx* ctx, const void* ptr, uint64_t rows, uint64_t cols,
                         uint32_t box_rows, bool u8 = false) {
  auto key = std::make_tuple(ptr, rows, cols, box_rows | (u8 ? 0x10000u : 0u));
  auto it = ctx->maps.find(key);
  if (it != ctx->maps.end()) return &it->second;
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return nullptr;
  CUtensorMap m;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (u8 ? 1 : 2)};
  cuuint32_t box[2] = {u8 ? 128u : 64u, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(&m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return nullptr;
  return &(ctx->maps[key] = m);
}

bool map_kv(CUtensorMap* m, void* base, uint64_t planes, uint64_t Lcap, uint64_t Dh) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {Dh, Lcap, planes};
  cuuint64_t strides[2] = {Dh * 2, Lcap * Dh * 2};
  cuuint32_t box[3] = {64, 128, 1};   // 64 head-dim columns x 128 keys (one attention tile half)
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q [positions][H][Dh] as a 3-D map whose box (64 columns, the G heads of a KV
// head, 128/G positions) is one 64-column half of a 128-row attention query
// tile; G must divide 128
bool map_q(CUtensorMap* m, void* q, uint64_t positions, uint64_t H, uint64_t Dh, uint32_t G) {
  if (G == 0 || 128 % G != 0) return false;
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {Dh, H, positions};
  cuuint64_t strides[2] = {Dh * 2, H * Dh * 2};
  cuuint32_t box[3] = {64, G, 128 / G};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int cdiv(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------------
// work plans
// ---------------------------------------------------------------------------

// splits of K that keep the most SMs busy (units = tiles * splits over
// whole waves of num_sms), fewer splits preferred on near ties
int pick_splits(int tiles, int kblocks, int num_sms, int max_splits) {
  if (tiles >= num_sms) return 1;
  int best = 1;
  double best_eff = 0.0;
  const int lim = std::min(max_splits, std::max(1, kblocks / 2));
  for (int s = 1; s <= lim; ++s) {
    const int units = tiles * s;
    const int waves = cdiv(units, num_sms);
    const double eff = (double)units / ((double)waves * num_sms);
    if (eff > best_eff + 0.02) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

GemmPlan plan_gemm(const dlm_ctx* ctx, int M, int N, int K, int epi) {
  GemmPlan p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.epi = epi;
  p.splits = 1;
  if (!ctx->bf16) {
    p.BN = 64;
    if (epi == EPI_F32) {
      const int tiles = cdiv(M, 64) * cdiv(N, 64);
      p.splits = pick_splits(tiles, cdiv(K, 16) / 4, ctx->num_sms, 8);
    }
    return p;
  }
  const int mt = cdiv(M, 128);
  if (epi == EPI_LM) {
    p.BN = mt > 1 ? 256 : 128;
    p.f8 = ctx->lm_f8 ? 1 : 0;
    p.f4 = ctx->lm_f4 ? 1 : 0;
    if (ctx->lm_f4) p.BN = 128;   // scale-factor columns fit tensor memory beside 2 x 128
    return p;
  }
  if (mt > 1) {
    // tensor-bound: K not split, so the projection epilogues can be fused
    // into the GEMM; 256-wide tiles: a 128 x 128 MMA step needs the whole
    // shared-memory bandwidth (measured ~6 against ~10 TFLOP/s per SM for
    // 128 x 256), so 128-wide tiles pay only when 256-wide ones leave most
    // SMs idle (fewer tiles than SMs and a clearly better fill)
    auto wave_eff = [&](int bn) {
      const int tiles = mt * cdiv(N, bn);
      return (double)tiles / ((double)cdiv(tiles, ctx->num_sms) * ctx->num_sms);
    };
    const bool under_one_wave = mt * cdiv(N, 256) < ctx->num_sms;
    p.BN = under_one_wave && wave_eff(128) > wave_eff(256) + 0.05 ? 128 : 256;
    return p;
  }
  // one M tile: weight-read bound; split K over as many CTAs as fit in one
  // wave (a second wave of short CTAs costs more pipeline fill than it saves)
  p.BN = 128;
  const int tiles = cdiv(N, p.BN);
  p.splits = tiles >= ctx->num_sms
                 ? 1
                 : std::max(1, std::min({16, ctx->num_sms / tiles, std::max(1, cdiv(K, 64) / 2)}));
  return p;
}

// Split plan of the attention.  For each CTA shape (128 query rows, or 256
// = two row tiles of the same KV head when it has that many rows) and every
// split count (with the smallest chunk of whole 128-key tiles that gives it)
// the CTAs are list-scheduled in launch order (split fastest) onto the SMs
// with a per-CTA and a per-tile time; ragged prefixes (lens, host) are taken
// as they are.  Up to 16 splits of 128-row CTAs may combine inside a
// thread-block cluster (an exchange cost per CTA) when the whole grid fits in
// one wave of resident clusters; otherwise splits write partials for the
// combine kernel (a write cost per CTA, the kernel, a cost per partial).
// Costs in microseconds, from B200 measurements: a 128-row tile of 128 keys
// takes ~1.2 us in a lone CTA and ~1.6 us when every SM streams K/V; a
// 256-row CTA reads each tile once for both row tiles (L2 already catches the
// second 128-row tile's reads) and takes ~2.65 us per tile pair.
// max_part_slots > 0 bounds the partial row slots (B * Hkv * nsplit * R) of
// plans that combine through the combine kernel; one split (no partials) and
// cluster plans always qualify.
AttnPlan plan_attention(const dlm_ctx* ctx, int B, int C, const int* lens, int max_len_all,
                        long max_part_slots = 0) {
  AttnPlan a{};
  a.B = B;
  a.C = C;
  a.G = ctx->md.H / ctx->md.Hkv;
  a.R = a.G * C;
  a.rtiles = cdiv(a.R, 128);
  const int Hkv = ctx->md.Hkv;
  const int sms = std::min(std::max(ctx->num_sms, 1), 1024);
  const int max_keys = max_len_all + C;
  const int max_tiles = cdiv(max_keys, 128);
  // the combine kernel: ~30 us after the attention for the batched shape's
  // 512 partial row tiles (device timeline), against the same attention with
  // one split and no partials
  const double t_xchg = 1.5, t_pw = 1.5, t_comb = 4.0, t_part = 0.05;
  double best = -1.0;
  double sm_free[1024];   // no heap allocation: this also runs inside dlm_attention_noalloc
  // diagnostic switch: DLM_ATTN_CLUSTER=0 keeps every split plan on the
  // partials + combine kernel path
  const char* cl_env = std::getenv("DLM_ATTN_CLUSTER");
  const bool cluster_ok = cl_env == nullptr || std::strcmp(cl_env, "0") != 0;
  // diagnostic switch: DLM_ATTN_TILES=k plans only chunks of k key tiles
  const char* ct_env = std::getenv("DLM_ATTN_TILES");
  const int only_ct = ct_env != nullptr ? std::atoi(ct_env) : 0;
  // diagnostic switch: DLM_ATTN_ROWS=128 or 256 plans only that CTA shape
  const char* rows_env = std::getenv("DLM_ATTN_ROWS");
  const int only_rows = rows_env != nullptr ? std::atoi(rows_env) : 0;
  for (int rows = 128; rows <= 256; rows += 128) {
    if (rows == 256 && a.rtiles < 2) continue;          // one row tile: nothing to pair
    if (only_rows > 0 && rows != only_rows && !(only_rows == 256 && a.rtiles < 2)) continue;
    const int ytiles = rows == 256 ? cdiv(a.rtiles, 2) : a.rtiles;   // CTAs per split
    // measured (device timeline): a 128-row tile ~1.2 us alone, ~1.6 us with
    // every SM streaming; a 256-row tile pair ~2.65 us -- the same per-row
    // rate, so the wider CTA wins only where it saves CTAs
    const double t_tile = rows == 256 ? 2.9 : 1.5;
    const double t_cta = rows == 256 ? 4.0 : 3.0;
    int last_nsplit = 0;
    for (int ct = 1; ct <= max_tiles; ++ct) {
      if (only_ct > 0 && ct != std::min(only_ct, max_tiles)) continue;
      const int chunk = ct * 128;
      const int nsplit = cdiv(max_keys, chunk);
      if (nsplit > 64) continue;   // the combine kernel holds up to 64 splits
      if (nsplit == last_nsplit) continue;   // a larger chunk for the same split count
      last_nsplit = nsplit;
      const long ctas = (long)B * Hkv * ytiles * nsplit;
      int cl = 1;
      if (rows == 128 && nsplit > 1 && nsplit <= 16 && cluster_ok) {
        const int cap = attn_cluster_capacity(nsplit);
        if (cap > 0 && ctas <= (long)cap * nsplit) cl = nsplit;
      }
      if (cl == 1 && nsplit > 1 && max_part_slots > 0 &&
          (long)B * Hkv * nsplit * a.R > max_part_slots)
        continue;   // the partials would not fit the caller's fixed scratch
      const double per_cta =
          t_cta + (cl > 1 ? t_xchg : (nsplit > 1 ? t_pw * rows / 128 : 0.0));
      // SMs as a min-heap of finish times (negated for the max-heap functions)
      std::fill(sm_free, sm_free + sms, 0.0);
      long partials = 0;
      double makespan = 0.0;
      for (int bg = 0; bg < B * Hkv; ++bg) {
        const int keys = (lens ? lens[bg / Hkv] : max_len_all) + C;
        for (int rt = 0; rt < ytiles; ++rt) {
          for (int sp = 0; sp < nsplit; ++sp) {
            const int k0 = sp * chunk;
            if (k0 >= keys && cl == 1) continue;   // exits at once
            const int tiles = k0 < keys ? cdiv(std::min(chunk, keys - k0), 128) : 0;
            std::pop_heap(sm_free, sm_free + sms);   // earliest free SM to the back
            sm_free[sms - 1] -= per_cta + tiles * t_tile;
            makespan = std::max(makespan, -sm_free[sms - 1]);
            std::push_heap(sm_free, sm_free + sms);
            partials += rows / 128;
          }
        }
      }
      const double cost = makespan + (nsplit > 1 && cl == 1 ? t_comb + t_part * partials : 0.0);
      if (best < 0.0 || cost < best - 1e-9) {
        best = cost;
        a.chunk = chunk;
        a.nsplit = nsplit;
        a.cluster = cl;
        a.rows = rows;
      }
    }
  }
  if (best < 0.0) {
    // nothing qualified (a forced chunk size whose partials do not fit the
    // caller's scratch): one split of 128-row CTAs needs no partials
    a.chunk = max_tiles * 128;
    a.nsplit = 1;
    a.cluster = 1;
    a.rows = 128;
  }
  return a;
}

// plan_attention, remembered per (batch, canvas, prefix lengths)
AttnPlan plan_attention_cached(dlm_ctx* ctx, int B, int C, int max_len_all) {
  std::vector<int> key(ctx->lens_h.begin(), ctx->lens_h.begin() + B);
  key.push_back(B);
  key.push_back(C);
  key.push_back(max_len_all);
  auto it = ctx->plans.find(key);
  if (it != ctx->plans.end()) return it->second;
  const AttnPlan ap = plan_attention(ctx, B, C, ctx->lens_h.data(), max_len_all);
  if (ctx->plans.size() > 256) ctx->plans.clear();
  ctx->plans.emplace(std::move(key), ap);
  return ap;
}

int max_len(const dlm_ctx* ctx, int batch) {
  int m = 0;
  for (int b = 0; b < batch; ++b) m = std::max(m, ctx->lens_h[b]);
  return m;
}

int ensure_attn_scratch(dlm_ctx* ctx, const AttnPlan& ap) {
  if (ap.nsplit <= 1 || ap.cluster > 1) return DLM_OK;
  const size_t slots = (size_t)ap.B * ctx->md.Hkv * ap.nsplit * ap.R;
  if (slots * ctx->md.Dh > ctx->opart_floats) {
    if (ctx->opart) {
      cudaFree(ctx->opart);
      ctx->owned.erase(std::find(ctx->owned.begin(), ctx->owned.end(), (void*)ctx->opart));
      ctx->opart = nullptr;
    }
    if (int rc = dalloc(ctx, &ctx->opart, slots * ctx->md.Dh * sizeof(float))) return rc;
    ctx->opart_floats = slots * ctx->md.Dh;
  }
  if (slots > ctx->ml_count) {
    if (ctx->ml) {
      cudaFree(ctx->ml);
      ctx->owned.erase(std::find(ctx->owned.begin(), ctx->owned.end(), (void*)ctx->ml));
      ctx->ml = nullptr;
    }
    if (int rc = dalloc(ctx, &ctx->ml, slots * sizeof(float2))) return rc;
    ctx->ml_count = slots;
  }
  return DLM_OK;
}

// ---------------------------------------------------------------------------
// validation
// ---------------------------------------------------------------------------

int check_params(dlm_ctx* ctx, const dlm_sampler_params* p, int batch) {
  if (p == nullptr) return fail(ctx, DLM_EINVAL, "params is NULL");
  if (batch < 1 || batch > ctx->d.max_batch)
    return fail(ctx, DLM_EINVAL, "batch must be in [1, max_batch]");
  if (p->canvas < 1 || p->canvas > ctx->d.max_canvas)
    return fail(ctx, DLM_EINVAL, "canvas must be in [1, max_canvas]");
  if (p->steps < 1) return fail(ctx, DLM_EINVAL, "steps must be >= 1");
  if (!(p->threshold >= 0.0f)) return fail(ctx, DLM_EINVAL, "threshold must be >= 0");
  if (p->corruption != DLM_MASK && p->corruption != DLM_UNIFORM)
    return fail(ctx, DLM_EINVAL, "corruption must be DLM_MASK or DLM_UNIFORM");
  if (p->editing != 0 && p->editing != 1) return fail(ctx, DLM_EINVAL, "editing must be 0 or 1");
  if (p->editing && !(p->editing_threshold == p->editing_threshold))
    return fail(ctx, DLM_EINVAL, "editing_threshold must be a number");
  if (p->corruption == DLM_MASK && (ctx->d.mask_id < 0 || ctx->d.mask_id >= ctx->d.vocab))
    return fail(ctx, DLM_EINVAL, "mask corruption needs mask_id in [0, vocab)");
  if (!(p->temperature >= 0.0f)) return fail(ctx, DLM_EINVAL, "temperature must be >= 0");
  if (p->entropy_bound >= 0.0f && !(p->t_min > 0.0f && p->t_max >= p->t_min))
    return fail(ctx, DLM_EINVAL, "entropy bound needs 0 < t_min <= t_max");
  if (p->stop_entropy > 0.0f && p->stability_steps < 0)
    return fail(ctx, DLM_EINVAL, "adaptive stopping needs stability_steps >= 0");
  return DLM_OK;
}

int check_canvas(dlm_ctx* ctx, const dlm_canvas* c, const dlm_sampler_params* p) {
  if (c == nullptr || !c->tokens || !c->committed || !c->step || !c->done || !c->eos_pos)
    return fail(ctx, DLM_EINVAL, "canvas buffers must all be non-NULL");
  if (p != nullptr && p->stop_entropy > 0.0f && (!c->prev_cand || !c->stable))
    return fail(ctx, DLM_EINVAL, "adaptive stopping needs canvas prev_cand and stable");
  return DLM_OK;
}

LmEpi make_epi(const dlm_ctx* ctx, const dlm_sampler_params* p, const dlm_canvas* c) {
  LmEpi e{};
  e.V = ctx->d.vocab;
  e.mask_id = p->corruption == DLM_MASK ? ctx->d.mask_id : -1;
  e.C = p->canvas;
  e.S = p->steps;
  e.t_max = p->t_max;
  e.t_min = p->t_min;
  if (p->entropy_bound >= 0.0f) {
    e.mode = LM_SAMPLE_ANNEAL;
  } else if (p->temperature > 0.0f) {
    e.mode = LM_SAMPLE_FIXED;
    e.inv_temp = 1.0f / p->temperature;
  } else {
    e.mode = LM_GREEDY;
  }
  e.seed_lo = (uint32_t)(p->seed & 0xFFFFFFFFull);
  e.seed_hi = (uint32_t)(p->seed >> 32);
  e.step = c->step;
  return e;
}

SelectArgs make_select(const dlm_ctx* ctx, const dlm_sampler_params* p, int batch) {
  SelectArgs a{};
  a.B = batch;
  a.C = p->canvas;
  a.S = p->steps;
  a.V = ctx->d.vocab;
  a.quota = p->quota > 0 ? p->quota : cdiv(p->canvas, p->steps);
  a.threshold = p->threshold;
  a.eb = p->entropy_bound >= 0.0f;
  a.bound = p->entropy_bound;
  a.uniform = p->corruption == DLM_UNIFORM;
  a.mask_id = ctx->d.mask_id;
  a.eos_id = ctx->d.eos_id;
  a.seed_lo = (uint32_t)(p->seed & 0xFFFFFFFFull);
  a.seed_hi = (uint32_t)(p->seed >> 32);
  a.stability_steps = p->stability_steps;
  a.stop_entropy = p->stop_entropy;
  a.editing = p->editing;
  a.edit_thr = p->editing_threshold;
  return a;
}

// one GEMM through the engine of the model's element type
int run_gemm(dlm_ctx* ctx, const void* A, const void* B, int Brows, const GemmPlan& plan,
             const GemmIO& io_in, cudaStream_t st) {
  cudaError_t e;
  GemmIO io = io_in;
  // the failure-detection hook applies to launches issued directly, never to
  // a graph being captured (a captured launch would starve on every replay)
  if (ctx->withhold_gemms > 0 && ctx->bf16 && st != ctx->cap) {
    io.withhold_loads = 1;
    --ctx->withhold_gemms;
  }
  if (ctx->bf16) {
    // 8- and 4-bit operands are mapped as bytes: K bytes (e4m3) or K / 2 (NVFP4)
    const bool u8 = plan.f8 != 0 || plan.f4 != 0;
    const uint64_t cols = plan.f4 ? (uint64_t)plan.K / 2 : (uint64_t)plan.K;
    const CUtensorMap* ta =
        map2d(ctx, A, (uint64_t)ctx->Mmax, cols, (uint32_t)gemm_tc_a_rows(plan.M), u8);
    const CUtensorMap* tb = map2d(ctx, B, (uint64_t)Brows, cols, (uint32_t)plan.BN, u8);
    if (ta == nullptr || tb == nullptr)
      return fail(ctx, DLM_ECUDA, "cuTensorMapEncodeTiled failed");
    e = gemm_tc(*ta, *tb, plan, io, ctx->num_sms, st);
  } else {
    e = gemm_f32((const float*)A, (const float*)B, plan, io, st);
  }
  if (e != cudaSuccess) return cuda_fail(ctx, "gemm launch", e);
  ++ctx->launches;
  return DLM_OK;
}

// record the measurement event of `stage` (begin or end) for the current step
int stage_event(dlm_ctx* ctx, int stage, bool end, cudaStream_t st) {
  if (ctx->ev_stage != stage || ctx->ev.empty()) return DLM_OK;
  const int pairs = (int)ctx->ev.size() / 2;
  // external: under stream capture the record becomes an event-record node of the graph
  cudaError_t e = cudaEventRecordWithFlags(ctx->ev[2 * (ctx->ev_step % pairs) + (end ? 1 : 0)],
                                           st, cudaEventRecordExternal);
  if (e != cudaSuccess) return cuda_fail(ctx, "cudaEventRecord (stage events)", e);
  return DLM_OK;
}

#define STAGE(s, end)                                                  \
  do {                                                                 \
    if (int rc_ = stage_event(ctx, (s), (end), st)) return rc_;         \
  } while (0)

// destinations of the fused projection epilogues
ProjEpi proj_epi(const dlm_ctx* ctx, int C) {
  ProjEpi pe;
  pe.H = ctx->md.H;
  pe.Hkv = ctx->md.Hkv;
  pe.Dh = ctx->md.Dh;
  pe.Lcap = ctx->Lcap;
  pe.C = C;
  pe.lens = ctx->lens_d;
  pe.rope = ctx->d.rope_theta > 0.0f ? ctx->rope : nullptr;
  pe.q = ctx->q;
  pe.kcache = ctx->kc;
  pe.vcache = ctx->vc;
  pe.x = ctx->x;
  pe.y = ctx->y;
  return pe;
}

// the kernel sequence of one denoising step
int enqueue_step(dlm_ctx* ctx, const dlm_canvas* c, int batch, const dlm_sampler_params* p,
                 dlm_canvas_stats* stats, const AttnPlan& ap, cudaStream_t st) {
  const ModelDims& md = ctx->md;
  const int C = p->canvas;
  const int rows = batch * C;
  cudaError_t e;
  // a1: embedding gather (+ count of unfinished canvases)
  STAGE(DLM_STAGE_EMBED, false);
  e = embed_rows(md, c->tokens, ctx->emb, ctx->x, rows, C, batch, c->done, ctx->n_active,
                 ctx->err, st);
  if (e != cudaSuccess) return cuda_fail(ctx, "embed", e);
  ++ctx->launches;
  STAGE(DLM_STAGE_EMBED, true);
  // a2: fused QKV projection, RoPE, q and canvas K/V into the cache
  STAGE(DLM_STAGE_QKV, false);
  {
    GemmPlan pl = plan_gemm(ctx, rows, ctx->Nqkv, md.d, EPI_F32);
    GemmIO io;
    io.out = ctx->part;
    io.n_active = ctx->n_active;
    io.err = ctx->err;
    io.trace_kind = TRACE_QKV_GEMM;
    const bool fused = ctx->bf16 && pl.splits == 1 && pl.BN >= 128 && cdiv(rows, 128) > 1;
    if (fused) {
      pl.epi = EPI_QKV;
      io.done = c->done;
      io.proj = proj_epi(ctx, C);
    }
    if (int rc = run_gemm(ctx, ctx->x, ctx->w_qkv, ctx->Nqkv, pl, io, st)) return rc;
    if (!fused) {
      e = qkv_epilogue(md, ctx->part, pl.splits, rows, C, -1, 0, ctx->lens_d, ctx->rope, ctx->q,
                       ctx->kc, ctx->vc, c->done, ctx->n_active, ctx->err, st);
      if (e != cudaSuccess) return cuda_fail(ctx, "qkv epilogue", e);
      ++ctx->launches;
    }
  }
  STAGE(DLM_STAGE_QKV, true);
  // a3: attention over [prefix ; canvas]
  STAGE(DLM_STAGE_ATTENTION, false);
  if (ctx->bf16) {
    e = attention_bf16(md, ap, ctx->tmK, ctx->tmV, ctx->has_tmQ ? &ctx->tmQ : nullptr, ctx->q,
                       ctx->o, ctx->opart, ctx->ml,
                       ctx->lens_d, c->done, ctx->n_active, ctx->err, st);
    ctx->launches += ap.nsplit > 1 && ap.cluster <= 1 ? 2 : 1;
  } else {
    e = attention_f32(md, batch, C, (const float*)ctx->q, (const float*)ctx->kc,
                      (const float*)ctx->vc, (float*)ctx->o, ctx->lens_d, c->done,
                      ctx->n_active, ctx->err, st);
    ++ctx->launches;
  }
  if (e != cudaSuccess) return cuda_fail(ctx, "attention", e);
  STAGE(DLM_STAGE_ATTENTION, true);
  // a4: output projection + residual
  STAGE(DLM_STAGE_WO, false);
  {
    GemmPlan pl = plan_gemm(ctx, rows, md.d, md.H * md.Dh, EPI_F32);
    GemmIO io;
    io.out = ctx->part;
    io.n_active = ctx->n_active;
    io.err = ctx->err;
    io.trace_kind = TRACE_WO_GEMM;
    const bool fused = ctx->bf16 && pl.splits == 1 && pl.BN >= 128 && cdiv(rows, 128) > 1;
    if (fused) {
      pl.epi = EPI_RESID;
      io.done = c->done;
      io.proj = proj_epi(ctx, C);
    }
    if (int rc = run_gemm(ctx, ctx->o, ctx->w_o, md.d, pl, io, st)) return rc;
    if (!fused) {
      e = wo_epilogue(md, ctx->part, pl.splits, rows, C, ctx->x, ctx->y, c->done, ctx->n_active,
                      st);
      if (e != cudaSuccess) return cuda_fail(ctx, "wo epilogue", e);
      ++ctx->launches;
    }
  }
  STAGE(DLM_STAGE_WO, true);
  // a5: LM head with the fused vocabulary reduction
  GemmPlan pl = plan_gemm(ctx, rows, md.V, md.d, EPI_LM);
  STAGE(DLM_STAGE_LM_HEAD, false);
  {
    GemmIO io;
    io.part = ctx->lmpart;
    io.epi = make_epi(ctx, p, c);
    io.done = c->done;
    io.n_active = ctx->n_active;
    io.err = ctx->err;
    io.trace_kind = TRACE_LM_HEAD;
    if (ctx->lm_f4) {
      // NVFP4 head: the rows are quantised first (elements, block scales, row
      // scales); block scales enter the MMA, row scales the epilogue
      e = quantize_rows_nvfp4(ctx->y, rows, md.d, ctx->yq, ctx->y_sf, ctx->s_y, C, c->done,
                              ctx->n_active, st);
      if (e != cudaSuccess) return cuda_fail(ctx, "quantize rows (NVFP4)", e);
      ++ctx->launches;
      io.epi.row_scale = ctx->s_y;
      io.epi.col_scale = ctx->s_lm;
      io.sfa = ctx->y_sf;
      io.sfb = ctx->lm_sf;
      if (int rc = run_gemm(ctx, ctx->yq, ctx->w_lm_q, md.V, pl, io, st)) return rc;
    } else if (ctx->lm_f8) {
      // e4m3 head: the rows are quantised first, the scales enter the epilogue
      e = quantize_rows_e4m3(ctx->y, rows, md.d, ctx->yq, ctx->s_y, C, c->done, ctx->n_active,
                             st);
      if (e != cudaSuccess) return cuda_fail(ctx, "quantize rows", e);
      ++ctx->launches;
      io.epi.row_scale = ctx->s_y;
      io.epi.col_scale = ctx->s_lm;
      if (int rc = run_gemm(ctx, ctx->yq, ctx->w_lm_q, md.V, pl, io, st)) return rc;
    } else {
      if (int rc = run_gemm(ctx, ctx->y, ctx->w_lm, md.V, pl, io, st)) return rc;
    }
  }
  STAGE(DLM_STAGE_LM_HEAD, true);
  // a6 + a7: cross-tile reduction, then commit / re-noise, one launch
  const int n_part = ctx->bf16 ? gemm_tc_lm_partials(pl, ctx->num_sms) : cdiv(md.V, pl.BN);
  STAGE(DLM_STAGE_COMMIT, false);
  e = commit_step(make_select(ctx, p, batch), c->tokens, c->committed, c->step, c->done,
                  c->eos_pos, c->prev_cand, c->stable, ctx->lmpart, n_part, ctx->cand, ctx->conf,
                  ctx->ent, stats, ctx->n_active, ctx->err, st);
  if (e != cudaSuccess) return cuda_fail(ctx, "commit", e);
  ++ctx->launches;
  STAGE(DLM_STAGE_COMMIT, true);
  ++ctx->ev_step;
  return DLM_OK;
}

// The clean pass over finished tokens of every sequence of the batch: K/V
// at positions len_b .. len_b+C-1 from the tokens themselves, then len_b += C.
int enqueue_clean_pass(dlm_ctx* ctx, const int32_t* tokens, int batch, int C, cudaStream_t st) {
  const ModelDims& md = ctx->md;
  const int rows = batch * C;
  cudaError_t e = embed_rows(md, tokens, ctx->emb, ctx->x, rows, C, batch, nullptr, nullptr,
                             ctx->err, st);
  if (e != cudaSuccess) return cuda_fail(ctx, "embed (clean pass)", e);
  GemmPlan pl = plan_gemm(ctx, rows, ctx->Nqkv, md.d, EPI_F32);
  GemmIO io;
  io.out = ctx->part;
  io.err = ctx->err;
  const bool fused = ctx->bf16 && pl.splits == 1 && pl.BN >= 128 && cdiv(rows, 128) > 1;
  if (fused) {
    pl.epi = EPI_QKV;
    io.proj = proj_epi(ctx, C);
  }
  if (int rc = run_gemm(ctx, ctx->x, ctx->w_qkv, ctx->Nqkv, pl, io, st)) return rc;
  if (!fused) {
    e = qkv_epilogue(md, ctx->part, pl.splits, rows, C, -1, 0, ctx->lens_d, ctx->rope, ctx->q,
                     ctx->kc, ctx->vc, nullptr, nullptr, ctx->err, st);
    if (e != cudaSuccess) return cuda_fail(ctx, "qkv epilogue (clean pass)", e);
  }
  e = add_len_all(ctx->lens_d, batch, C, st);
  if (e != cudaSuccess) return cuda_fail(ctx, "add_len_all", e);
  for (int b = 0; b < batch; ++b) ctx->lens_h[b] += C;
  return DLM_OK;
}

size_t part_floats_needed(const dlm_ctx* ctx) {
  size_t need = 0;
  const ModelDims& md = ctx->md;
  std::vector<int> Ms;
  for (int m = 1; m <= ctx->Mmax; m = (m < 128 ? m * 2 : m + 128)) Ms.push_back(m);
  Ms.push_back(ctx->Mmax);
  for (int M : Ms) {
    const int uses[3][2] = {{ctx->Nqkv, md.d}, {md.d, md.H * md.Dh}, {2 * md.Hkv * md.Dh, md.d}};
    for (auto& u : uses) {
      GemmPlan pl = plan_gemm(ctx, M, u[0], u[1], EPI_F32);
      need = std::max(need, (size_t)pl.splits * M * u[0]);
    }
  }
  return need;
}

void destroy_graphs(dlm_ctx* ctx) {
  for (auto& g : ctx->graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  ctx->graphs.clear();
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================

extern "C" {

int dlm_create(const dlm_model_desc* desc, const dlm_weights* w, dlm_ctx** out) {
  g_create_error.clear();
  if (out == nullptr) return fail(nullptr, DLM_EINVAL, "out is NULL");
  *out = nullptr;
  if (desc == nullptr || w == nullptr) return fail(nullptr, DLM_EINVAL, "desc/weights NULL");
  const dlm_model_desc& d = *desc;
  if (d.dtype != DLM_F32 && d.dtype != DLM_BF16)
    return fail(nullptr, DLM_EINVAL, "dtype must be DLM_F32 or DLM_BF16");
  if (d.d_model <= 0 || d.n_heads <= 0 || d.n_kv_heads <= 0 || d.vocab <= 0 || d.head_dim <= 0)
    return fail(nullptr, DLM_EINVAL, "model dimensions must be positive");
  if (d.n_heads % d.n_kv_heads != 0)
    return fail(nullptr, DLM_EINVAL, "n_heads must be a multiple of n_kv_heads");
  if (d.dtype == DLM_BF16 && (d.head_dim != 128 || d.d_model % 64 != 0))
    return fail(nullptr, DLM_EINVAL, "bf16 model needs head_dim 128 and d_model % 64 == 0");
  if (d.dtype == DLM_F32 && !(d.head_dim == 32 || d.head_dim == 64 || d.head_dim == 128))
    return fail(nullptr, DLM_EINVAL, "fp32 model needs head_dim 32, 64 or 128");
  if (d.dtype == DLM_F32 && d.d_model % 4 != 0)
    return fail(nullptr, DLM_EINVAL, "fp32 model needs d_model % 4 == 0");
  if (d.mask_id >= d.vocab || d.eos_id >= d.vocab)
    return fail(nullptr, DLM_EINVAL, "mask_id / eos_id must be < vocab");
  if (d.max_batch < 1 || d.max_prefix < 0 || d.max_canvas < 1 || d.max_canvas > 1024)
    return fail(nullptr, DLM_EINVAL, "need max_batch >= 1, max_prefix >= 0, 1 <= max_canvas <= 1024");
  if (!w->emb || !w->w_q || !w->w_k || !w->w_v || !w->w_o || !w->w_lm)
    return fail(nullptr, DLM_EINVAL, "every weight pointer must be non-NULL");
  if (d.lm_quant != DLM_LM_MODEL && d.lm_quant != DLM_LM_E4M3 && d.lm_quant != DLM_LM_NVFP4)
    return fail(nullptr, DLM_EINVAL, "lm_quant must be DLM_LM_MODEL, DLM_LM_E4M3 or DLM_LM_NVFP4");
  if (d.lm_quant == DLM_LM_E4M3 && (d.dtype != DLM_BF16 || d.d_model % 16 != 0))
    return fail(nullptr, DLM_EINVAL, "the e4m3 LM head needs a bf16 model with d_model % 16 == 0");
  if (d.lm_quant == DLM_LM_NVFP4 && (d.dtype != DLM_BF16 || d.d_model % 256 != 0))
    return fail(nullptr, DLM_EINVAL,
                "the NVFP4 LM head needs a bf16 model with d_model % 256 == 0");

  dlm_ctx* ctx = new dlm_ctx();
  ctx->d = d;
  ctx->bf16 = d.dtype == DLM_BF16;
  ctx->lm_f8 = d.lm_quant == DLM_LM_E4M3;
  ctx->lm_f4 = d.lm_quant == DLM_LM_NVFP4;
  ctx->es = ctx->bf16 ? 2 : 4;
  cudaGetDevice(&ctx->dev);
  cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->dev);
  ctx->Lcap = d.max_prefix + d.max_canvas;
  ctx->md = ModelDims{d.d_model, d.n_heads, d.n_kv_heads, d.head_dim, d.vocab, d.mask_id,
                      d.eos_id, ctx->Lcap, (int)ctx->es};
  ctx->Nqkv = (d.n_heads + 2 * d.n_kv_heads) * d.head_dim;
  ctx->Mmax = d.max_batch * d.max_canvas;
  ctx->emb = w->emb;
  ctx->w_o = w->w_o;
  ctx->w_lm = w->w_lm;
  ctx->lens_h.assign(d.max_batch, 0);

  auto bail = [&](int rc) {
    g_create_error = ctx->msg;
    dlm_destroy(ctx);
    return rc;
  };
  const size_t es = ctx->es;
  const size_t dm = d.d_model, qd = (size_t)d.n_heads * d.head_dim;
  const size_t kv_elems = (size_t)d.max_batch * d.n_kv_heads * ctx->Lcap * d.head_dim;
  int rc = DLM_OK;
  if ((rc = dalloc(ctx, &ctx->w_qkv, (size_t)ctx->Nqkv * dm * es))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->kc, kv_elems * es))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->vc, kv_elems * es))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->lens_d, d.max_batch * sizeof(int32_t)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->x, ctx->Mmax * dm * es))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->q, ctx->Mmax * qd * es))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->o, ctx->Mmax * qd * es))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->y, ctx->Mmax * dm * es))) return bail(rc);
  const int lm_tile = ctx->bf16 ? 128 : 64;
  if ((rc = dalloc(ctx, &ctx->lmpart,
                   (size_t)ctx->Mmax * cdiv(d.vocab, lm_tile) * kLmFields * sizeof(float))))
    return bail(rc);
  if ((rc = dalloc(ctx, &ctx->cand, ctx->Mmax * sizeof(int32_t)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->conf, ctx->Mmax * sizeof(float)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->ent, ctx->Mmax * sizeof(float)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->rope, (size_t)ctx->Lcap * (d.head_dim / 2) * sizeof(float2))))
    return bail(rc);
  if ((rc = dalloc(ctx, &ctx->n_active, 2 * sizeof(int)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->err, sizeof(int)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->h_tok, ctx->Mmax * sizeof(int32_t)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->h_com, ctx->Mmax))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->h_step, d.max_batch * sizeof(int32_t)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->h_done, d.max_batch))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->h_eos, d.max_batch * sizeof(int32_t)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->h_stats, d.max_batch * sizeof(dlm_canvas_stats)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->h_prev, ctx->Mmax * sizeof(int32_t)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->h_stable, d.max_batch * sizeof(int32_t)))) return bail(rc);
  ctx->part_floats = part_floats_needed(ctx);
  if ((rc = dalloc(ctx, &ctx->part, ctx->part_floats * sizeof(float)))) return bail(rc);
  if (ctx->lm_f8 || ctx->lm_f4) {
    // one byte per element (e4m3) or two elements per byte (NVFP4)
    const size_t row_bytes = ctx->lm_f4 ? dm / 2 : dm;
    ctx->s_lm_count = (size_t)cdiv(d.vocab, 256) * 256;   // whole tiles of either width
    if ((rc = dalloc(ctx, &ctx->w_lm_q, (size_t)d.vocab * row_bytes))) return bail(rc);
    if ((rc = dalloc(ctx, &ctx->s_lm, ctx->s_lm_count * sizeof(float)))) return bail(rc);
    if ((rc = dalloc(ctx, &ctx->yq, ctx->Mmax * row_bytes))) return bail(rc);
    if ((rc = dalloc(ctx, &ctx->s_y, ctx->Mmax * sizeof(float)))) return bail(rc);
  }
  if (ctx->lm_f4) {
    // block scales: [row block of 128][d / 64][512 bytes]
    ctx->lm_sf_bytes = (size_t)cdiv(d.vocab, 128) * (dm / 64) * 512;
    ctx->y_sf_bytes = (size_t)cdiv(ctx->Mmax, 128) * (dm / 64) * 512;
    if ((rc = dalloc(ctx, &ctx->lm_sf, ctx->lm_sf_bytes))) return bail(rc);
    if ((rc = dalloc(ctx, &ctx->y_sf, ctx->y_sf_bytes))) return bail(rc);
  }

  cudaError_t e = cudaSuccess;
  auto ck = [&](cudaError_t r, const char* what) {
    if (r != cudaSuccess && e == cudaSuccess) {
      e = r;
      cuda_fail(ctx, what, r);
    }
  };
  ck(cudaMemset(ctx->kc, 0, kv_elems * es), "memset K cache");
  ck(cudaMemset(ctx->vc, 0, kv_elems * es), "memset V cache");
  ck(cudaMemset(ctx->lens_d, 0, d.max_batch * sizeof(int32_t)), "memset lens");
  ck(cudaMemset(ctx->x, 0, ctx->Mmax * dm * es), "memset x");
  ck(cudaMemset(ctx->o, 0, ctx->Mmax * qd * es), "memset o");
  ck(cudaMemset(ctx->y, 0, ctx->Mmax * dm * es), "memset y");
  ck(cudaMemset(ctx->err, 0, sizeof(int)), "memset err");
  // fused [W_q ; W_k ; W_v]
  const size_t qb = qd * dm * es, kvb = (size_t)d.n_kv_heads * d.head_dim * dm * es;
  ck(cudaMemcpy(ctx->w_qkv, w->w_q, qb, cudaMemcpyDeviceToDevice), "copy w_q");
  ck(cudaMemcpy((uint8_t*)ctx->w_qkv + qb, w->w_k, kvb, cudaMemcpyDeviceToDevice), "copy w_k");
  ck(cudaMemcpy((uint8_t*)ctx->w_qkv + qb + kvb, w->w_v, kvb, cudaMemcpyDeviceToDevice),
     "copy w_v");
  if (d.rope_theta > 0.0f)
    ck(rope_table_init(ctx->rope, ctx->Lcap, d.head_dim, (double)d.rope_theta, nullptr),
       "rope table");
  if (ctx->lm_f4) {
    ck(cudaMemset(ctx->s_lm, 0, ctx->s_lm_count * sizeof(float)), "memset LM scales");
    ck(cudaMemset(ctx->yq, 0, ctx->Mmax * dm / 2), "memset quantised rows");
    ck(cudaMemset(ctx->s_y, 0, ctx->Mmax * sizeof(float)), "memset row scales");
    ck(cudaMemset(ctx->lm_sf, 0, ctx->lm_sf_bytes), "memset LM block scales");
    ck(cudaMemset(ctx->y_sf, 0, ctx->y_sf_bytes), "memset row block scales");
    ck(quantize_rows_nvfp4(w->w_lm, d.vocab, d.d_model, ctx->w_lm_q, ctx->lm_sf, ctx->s_lm, 1,
                           nullptr, nullptr, nullptr),
       "quantise LM head (NVFP4)");
  }
  if (ctx->lm_f8) {
    ck(cudaMemset(ctx->s_lm, 0, ctx->s_lm_count * sizeof(float)), "memset LM scales");
    ck(cudaMemset(ctx->yq, 0, ctx->Mmax * dm), "memset quantised rows");
    ck(cudaMemset(ctx->s_y, 0, ctx->Mmax * sizeof(float)), "memset row scales");
    ck(quantize_rows_e4m3(w->w_lm, d.vocab, d.d_model, ctx->w_lm_q, ctx->s_lm, 1, nullptr,
                          nullptr, nullptr),
       "quantise LM head");
  }
  ck(cudaStreamCreateWithFlags(&ctx->cap, cudaStreamNonBlocking), "capture stream");
  ck(cudaDeviceSynchronize(), "create sync");
  if (e != cudaSuccess) return bail(DLM_ECUDA);
  if (ctx->bf16) {
    const uint64_t planes = (uint64_t)d.max_batch * d.n_kv_heads;
    if (!map_kv(&ctx->tmK, ctx->kc, planes, ctx->Lcap, d.head_dim) ||
        !map_kv(&ctx->tmV, ctx->vc, planes, ctx->Lcap, d.head_dim))
      return bail(fail(ctx, DLM_ECUDA, "cuTensorMapEncodeTiled (KV cache) failed"));
    ctx->has_tmQ = map_q(&ctx->tmQ, ctx->q, (uint64_t)ctx->Mmax, d.n_heads, d.head_dim,
                         (uint32_t)(d.n_heads / d.n_kv_heads));
  }
  *out = ctx;
  return DLM_OK;
}

void dlm_destroy(dlm_ctx* ctx) {
  if (ctx == nullptr) return;
  cudaDeviceSynchronize();
  destroy_graphs(ctx);
  if (ctx->cap) cudaStreamDestroy(ctx->cap);
  for (void* p : ctx->owned) cudaFree(p);
  delete ctx;
}

int dlm_kv_append(dlm_ctx* ctx, int seq, int n, const int32_t* tokens, const void* k,
                  const void* v, void* stream) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (seq < 0 || seq >= ctx->d.max_batch) return fail(ctx, DLM_EINVAL, "seq out of range");
  if (n < 0) return fail(ctx, DLM_EINVAL, "n must be >= 0");
  if (n == 0) return DLM_OK;
  if ((long)ctx->lens_h[seq] + n > ctx->d.max_prefix)
    return fail(ctx, DLM_ECAP, "KV capacity exceeded");
  cudaStream_t st = (cudaStream_t)stream;
  const ModelDims& md = ctx->md;
  if (tokens == nullptr) {
    if (k == nullptr || v == nullptr) return fail(ctx, DLM_EINVAL, "need tokens or k and v");
    CK(kv_copy_in(md, seq, n, k, v, ctx->lens_d, ctx->kc, ctx->vc, ctx->err, st));
    CK(add_len(ctx->lens_d, seq, n, st));
  } else {
    const int Nkv = 2 * md.Hkv * md.Dh;
    const void* wkv = (const uint8_t*)ctx->w_qkv + (size_t)md.H * md.Dh * md.d * ctx->es;
    for (int j0 = 0; j0 < n; j0 += ctx->Mmax) {
      const int rows = std::min(ctx->Mmax, n - j0);
      CK(embed_rows(md, tokens + j0, ctx->emb, ctx->x, rows, rows, 1, nullptr, nullptr, ctx->err,
                    st));
      GemmPlan pl = plan_gemm(ctx, rows, Nkv, md.d, EPI_F32);
      GemmIO io;
      io.out = ctx->part;
      io.err = ctx->err;
      if (int rc = run_gemm(ctx, ctx->x, wkv, Nkv, pl, io, st)) return rc;
      CK(qkv_epilogue(md, ctx->part, pl.splits, rows, rows, seq, md.H, ctx->lens_d, ctx->rope,
                      nullptr, ctx->kc, ctx->vc, nullptr, nullptr, ctx->err, st));
      CK(add_len(ctx->lens_d, seq, rows, st));
    }
  }
  ctx->lens_h[seq] += n;
  return DLM_OK;
}

int dlm_reset_kv(dlm_ctx* ctx, int seq) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (seq < 0 || seq >= ctx->d.max_batch) return fail(ctx, DLM_EINVAL, "seq out of range");
  ctx->lens_h[seq] = 0;
  CK(cudaMemset(ctx->lens_d + seq, 0, sizeof(int32_t)));
  return DLM_OK;
}

int dlm_kv_length(const dlm_ctx* ctx, int seq) {
  if (ctx == nullptr || seq < 0 || seq >= ctx->d.max_batch) return DLM_EINVAL;
  return ctx->lens_h[seq];
}

int dlm_canvas_init(dlm_ctx* ctx, const dlm_canvas* c, int batch, const dlm_sampler_params* p,
                    void* stream) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (int rc = check_params(ctx, p, batch)) return rc;
  if (int rc = check_canvas(ctx, c, p)) return rc;
  CK(canvas_init(ctx->md, batch, p->canvas, p->corruption, p->seed, c->tokens, c->committed,
                 c->step, c->done, c->eos_pos, c->prev_cand, c->stable, (cudaStream_t)stream));
  return DLM_OK;
}

int dlm_denoise_step(dlm_ctx* ctx, const dlm_canvas* c, int batch, const dlm_sampler_params* p,
                     dlm_canvas_stats* stats, void* stream) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (int rc = check_params(ctx, p, batch)) return rc;
  if (int rc = check_canvas(ctx, c, p)) return rc;
  AttnPlan ap = plan_attention_cached(ctx, batch, p->canvas, max_len(ctx, batch));
  if (ctx->bf16)
    if (int rc = ensure_attn_scratch(ctx, ap)) return rc;
  ctx->launches = 0;
  return enqueue_step(ctx, c, batch, p, stats, ap, (cudaStream_t)stream);
}

}  // extern "C"

namespace {

// `n_steps` denoising steps as one CUDA graph, captured once per
// configuration (pointers, sizes, parameters, attention plan, step count) and
// replayed on `stream`
int decode_steps_graph(dlm_ctx* ctx, const dlm_canvas* c, int batch, const dlm_sampler_params* p,
                       int n_steps, dlm_canvas_stats* stats, void* stream) {
  AttnPlan ap = plan_attention_cached(ctx, batch, p->canvas, max_len(ctx, batch));
  if (ctx->bf16)
    if (int rc = ensure_attn_scratch(ctx, ap)) return rc;
  // the graph bakes in pointers, sizes, parameters and the attention plan
  std::vector<uint8_t> key(sizeof(int) * 5 + sizeof(dlm_sampler_params) + sizeof(dlm_canvas) +
                           sizeof(void*) * 3 + ctx->ev.size() * sizeof(cudaEvent_t));
  uint8_t* kp = key.data();
  const int hdr[5] = {batch, ap.chunk, ap.nsplit, ctx->ev_stage, n_steps};
  const void* ptrs[3] = {stats, ctx->opart, ctx->ml};
  std::memcpy(kp, hdr, sizeof(hdr));
  kp += sizeof(hdr);
  dlm_sampler_params pc = *p;
  std::memcpy(kp, &pc, sizeof(pc));
  kp += sizeof(pc);
  std::memcpy(kp, c, sizeof(*c));
  kp += sizeof(*c);
  std::memcpy(kp, ptrs, sizeof(ptrs));
  kp += sizeof(ptrs);
  if (!ctx->ev.empty()) std::memcpy(kp, ctx->ev.data(), ctx->ev.size() * sizeof(cudaEvent_t));
  GraphEntry* ge = nullptr;
  for (auto& g : ctx->graphs)
    if (g.key == key) ge = &g;
  if (ge == nullptr) {
    if (ctx->graphs.size() >= 8) {
      cudaGraphExecDestroy(ctx->graphs.front().exec);
      ctx->graphs.erase(ctx->graphs.begin());
    }
    cudaGraph_t graph = nullptr;
    CK(cudaStreamBeginCapture(ctx->cap, cudaStreamCaptureModeThreadLocal));
    ctx->launches = 0;
    ctx->ev_step = 0;
    int rc = DLM_OK;
    for (int s = 0; s < n_steps && rc == DLM_OK; ++s)
      rc = enqueue_step(ctx, c, batch, p, stats, ap, ctx->cap);
    cudaError_t ce = cudaStreamEndCapture(ctx->cap, &graph);
    if (rc != DLM_OK) {
      if (graph) cudaGraphDestroy(graph);
      return rc;
    }
    if (ce != cudaSuccess) return cuda_fail(ctx, "cudaStreamEndCapture", ce);
    GraphEntry g;
    g.key = key;
    g.launches = ctx->launches / n_steps;
    ce = cudaGraphInstantiate(&g.exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ce != cudaSuccess) return cuda_fail(ctx, "cudaGraphInstantiate", ce);
    ctx->graphs.push_back(g);
    ge = &ctx->graphs.back();
  }
  ctx->launches = ge->launches;
  CK(cudaGraphLaunch(ge->exec, (cudaStream_t)stream));
  return DLM_OK;
}

}  // namespace

extern "C" {

int dlm_decode_block(dlm_ctx* ctx, const dlm_canvas* c, int batch, const dlm_sampler_params* p,
                     dlm_canvas_stats* stats, void* stream) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (int rc = check_params(ctx, p, batch)) return rc;
  if (int rc = check_canvas(ctx, c, p)) return rc;
  return decode_steps_graph(ctx, c, batch, p, p->steps, stats, stream);
}

int dlm_decode_steps(dlm_ctx* ctx, const dlm_canvas* c, int batch, const dlm_sampler_params* p,
                     int n_steps, dlm_canvas_stats* stats, void* stream) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (int rc = check_params(ctx, p, batch)) return rc;
  if (int rc = check_canvas(ctx, c, p)) return rc;
  if (n_steps < 1 || n_steps > p->steps)
    return fail(ctx, DLM_EINVAL, "n_steps must be in [1, params->steps]");
  return decode_steps_graph(ctx, c, batch, p, n_steps, stats, stream);
}

int dlm_attention_plan(dlm_ctx* ctx, int batch, int canvas, int* nsplit, int* chunk,
                       int* cluster, int* rows_per_cta) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (!nsplit || !chunk || !cluster || !rows_per_cta)
    return fail(ctx, DLM_EINVAL, "attention_plan: NULL output pointer");
  if (!ctx->bf16) return fail(ctx, DLM_EINVAL, "attention_plan: the fp32 model has no split plan");
  if (batch < 1 || batch > ctx->d.max_batch || canvas < 1 || canvas > ctx->d.max_canvas)
    return fail(ctx, DLM_EINVAL, "attention_plan: batch or canvas out of range");
  const AttnPlan ap = plan_attention_cached(ctx, batch, canvas, max_len(ctx, batch));
  *nsplit = ap.nsplit;
  *chunk = ap.chunk;
  *cluster = ap.cluster;
  *rows_per_cta = ap.rows;
  return DLM_OK;
}

int dlm_decode_block_host(dlm_ctx* ctx, int32_t* tokens, uint8_t* committed, int32_t* step,
                          uint8_t* done, int32_t* eos_pos, int batch,
                          const dlm_sampler_params* p, dlm_canvas_stats* stats, void* stream) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (int rc = check_params(ctx, p, batch)) return rc;
  if (!tokens || !committed || !step || !done || !eos_pos)
    return fail(ctx, DLM_EINVAL, "host canvas buffers must be non-NULL");
  cudaStream_t st = (cudaStream_t)stream;
  const size_t n = (size_t)batch * p->canvas;
  CK(cudaMemcpyAsync(ctx->h_tok, tokens, n * sizeof(int32_t), cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(ctx->h_com, committed, n, cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(ctx->h_step, step, batch * sizeof(int32_t), cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(ctx->h_done, done, batch, cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(ctx->h_eos, eos_pos, batch * sizeof(int32_t), cudaMemcpyHostToDevice, st));
  if (stats)
    CK(cudaMemcpyAsync(ctx->h_stats, stats, batch * sizeof(dlm_canvas_stats),
                       cudaMemcpyHostToDevice, st));
  // adaptive-stopping state starts fresh for every call
  CK(cudaMemsetAsync(ctx->h_prev, 0xFF, n * sizeof(int32_t), st));
  CK(cudaMemsetAsync(ctx->h_stable, 0, batch * sizeof(int32_t), st));
  dlm_canvas c{ctx->h_tok, ctx->h_com, ctx->h_step, ctx->h_done, ctx->h_eos, ctx->h_prev,
               ctx->h_stable};
  if (int rc = dlm_decode_block(ctx, &c, batch, p, stats ? ctx->h_stats : nullptr, stream))
    return rc;
  CK(cudaMemcpyAsync(tokens, ctx->h_tok, n * sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  CK(cudaMemcpyAsync(committed, ctx->h_com, n, cudaMemcpyDeviceToHost, st));
  CK(cudaMemcpyAsync(step, ctx->h_step, batch * sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  CK(cudaMemcpyAsync(done, ctx->h_done, batch, cudaMemcpyDeviceToHost, st));
  CK(cudaMemcpyAsync(eos_pos, ctx->h_eos, batch * sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  if (stats)
    CK(cudaMemcpyAsync(stats, ctx->h_stats, batch * sizeof(dlm_canvas_stats),
                       cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  return DLM_OK;
}

int dlm_generate(dlm_ctx* ctx, const dlm_canvas* c, int batch, const dlm_sampler_params* p,
                 int n_blocks, int eos_early_stop, int32_t* out_tokens, dlm_canvas_stats* stats,
                 int* blocks_done, void* stream) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (blocks_done) *blocks_done = 0;
  if (int rc = check_params(ctx, p, batch)) return rc;
  if (int rc = check_canvas(ctx, c, p)) return rc;
  if (n_blocks < 1 || out_tokens == nullptr)
    return fail(ctx, DLM_EINVAL, "generate needs n_blocks >= 1 and out_tokens");
  const int C = p->canvas;
  for (int b = 0; b < batch; ++b)
    if ((long)ctx->lens_h[b] + (long)n_blocks * C > ctx->d.max_prefix)
      return fail(ctx, DLM_ECAP, "prefix + n_blocks * canvas exceeds max_prefix");
  cudaStream_t st = (cudaStream_t)stream;
  std::vector<int32_t> eos(batch);
  for (int k = 0; k < n_blocks; ++k) {
    dlm_sampler_params pk = *p;
    pk.seed = p->seed + (unsigned long long)k;   // block k's random streams
    CK(canvas_init(ctx->md, batch, C, pk.corruption, pk.seed, c->tokens, c->committed, c->step,
                   c->done, c->eos_pos, c->prev_cand, c->stable, st));
    AttnPlan ap = plan_attention_cached(ctx, batch, C, max_len(ctx, batch));
    if (ctx->bf16)
      if (int rc = ensure_attn_scratch(ctx, ap)) return rc;
    ctx->launches = 0;
    for (int s = 0; s < pk.steps; ++s)
      if (int rc = enqueue_step(ctx, c, batch, &pk, stats, ap, st)) return rc;
    CK(cudaMemcpy2DAsync(out_tokens + (size_t)k * C, (size_t)n_blocks * C * sizeof(int32_t),
                         c->tokens, (size_t)C * sizeof(int32_t), (size_t)C * sizeof(int32_t),
                         batch, cudaMemcpyDeviceToDevice, st));
    if (int rc = enqueue_clean_pass(ctx, c->tokens, batch, C, st)) return rc;
    if (blocks_done) *blocks_done = k + 1;
    if (eos_early_stop) {
      CK(cudaMemcpyAsync(eos.data(), c->eos_pos, batch * sizeof(int32_t), cudaMemcpyDeviceToHost,
                         st));
      CK(cudaStreamSynchronize(st));
      bool all = true;
      for (int b = 0; b < batch; ++b) all = all && eos[b] >= 0;
      if (all) break;
    }
  }
  return DLM_OK;
}

int dlm_commit(dlm_ctx* ctx, const dlm_canvas* c, int batch, const dlm_sampler_params* p,
               const int32_t* cand, const float* conf, const float* entropy,
               dlm_canvas_stats* stats, void* stream) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (int rc = check_params(ctx, p, batch)) return rc;
  if (int rc = check_canvas(ctx, c, p)) return rc;
  if (!cand || !conf || !entropy) return fail(ctx, DLM_EINVAL, "cand/conf/entropy NULL");
  CK(commit_step(make_select(ctx, p, batch), c->tokens, c->committed, c->step, c->done,
                 c->eos_pos, c->prev_cand, c->stable, nullptr, 0, const_cast<int32_t*>(cand),
                 const_cast<float*>(conf), const_cast<float*>(entropy), stats, nullptr, ctx->err,
                 (cudaStream_t)stream));
  return DLM_OK;
}

int dlm_debug_buffer(dlm_ctx* ctx, int which, void** ptr, size_t* bytes) {
  if (ctx == nullptr || ptr == nullptr || bytes == nullptr) return DLM_EINVAL;
  const size_t M = ctx->Mmax, es = ctx->es, dm = ctx->d.d_model;
  const size_t qd = (size_t)ctx->d.n_heads * ctx->d.head_dim;
  const size_t kv = (size_t)ctx->d.max_batch * ctx->d.n_kv_heads * ctx->Lcap * ctx->d.head_dim;
  switch (which) {
    case DLM_BUF_X: *ptr = ctx->x; *bytes = M * dm * es; break;
    case DLM_BUF_Q: *ptr = ctx->q; *bytes = M * qd * es; break;
    case DLM_BUF_O: *ptr = ctx->o; *bytes = M * qd * es; break;
    case DLM_BUF_Y: *ptr = ctx->y; *bytes = M * dm * es; break;
    case DLM_BUF_CAND: *ptr = ctx->cand; *bytes = M * 4; break;
    case DLM_BUF_CONF: *ptr = ctx->conf; *bytes = M * 4; break;
    case DLM_BUF_ENTROPY: *ptr = ctx->ent; *bytes = M * 4; break;
    case DLM_BUF_K_CACHE: *ptr = ctx->kc; *bytes = kv * es; break;
    case DLM_BUF_V_CACHE: *ptr = ctx->vc; *bytes = kv * es; break;
    case DLM_BUF_LM_Q:
    case DLM_BUF_LM_SCALE:
    case DLM_BUF_Y_Q:
    case DLM_BUF_Y_SCALE: {
      if (!ctx->lm_f8 && !ctx->lm_f4)
        return fail(ctx, DLM_EINVAL, "the context has no low-bit LM head");
      const size_t row_bytes = ctx->lm_f4 ? dm / 2 : dm;
      if (which == DLM_BUF_LM_Q) {
        *ptr = ctx->w_lm_q;
        *bytes = (size_t)ctx->d.vocab * row_bytes;
      } else if (which == DLM_BUF_LM_SCALE) {
        *ptr = ctx->s_lm;
        *bytes = ctx->s_lm_count * 4;
      } else if (which == DLM_BUF_Y_Q) {
        *ptr = ctx->yq;
        *bytes = M * row_bytes;
      } else {
        *ptr = ctx->s_y;
        *bytes = M * 4;
      }
      break;
    }
    case DLM_BUF_LM_SF:
    case DLM_BUF_Y_SF:
      if (!ctx->lm_f4) return fail(ctx, DLM_EINVAL, "the context has no NVFP4 LM head");
      *ptr = which == DLM_BUF_LM_SF ? ctx->lm_sf : ctx->y_sf;
      *bytes = which == DLM_BUF_LM_SF ? ctx->lm_sf_bytes : ctx->y_sf_bytes;
      break;
    default: return fail(ctx, DLM_EINVAL, "unknown buffer id");
  }
  return DLM_OK;
}

int dlm_debug_logits(dlm_ctx* ctx, int batch, int canvas, float* logits, void* stream) {
  if (ctx == nullptr || logits == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (batch < 1 || canvas < 1 || (long)batch * canvas > ctx->Mmax)
    return fail(ctx, DLM_EINVAL, "batch * canvas out of range");
  const int rows = batch * canvas;
  GemmPlan pl = plan_gemm(ctx, rows, ctx->d.vocab, ctx->d.d_model, EPI_LM);
  pl.epi = EPI_F32;
  pl.splits = 1;
  GemmIO io;
  io.out = logits;
  io.err = ctx->err;
  if (ctx->lm_f4) {
    io.epi.row_scale = ctx->s_y;
    io.epi.col_scale = ctx->s_lm;
    io.sfa = ctx->y_sf;
    io.sfb = ctx->lm_sf;
    return run_gemm(ctx, ctx->yq, ctx->w_lm_q, ctx->d.vocab, pl, io, (cudaStream_t)stream);
  }
  if (ctx->lm_f8) {
    io.epi.row_scale = ctx->s_y;
    io.epi.col_scale = ctx->s_lm;
    return run_gemm(ctx, ctx->yq, ctx->w_lm_q, ctx->d.vocab, pl, io, (cudaStream_t)stream);
  }
  return run_gemm(ctx, ctx->y, ctx->w_lm, ctx->d.vocab, pl, io, (cudaStream_t)stream);
}

int dlm_check(dlm_ctx* ctx, void* stream) {
  if (ctx == nullptr) return DLM_EINVAL;
  CK(cudaStreamSynchronize((cudaStream_t)stream));
  int word = 0;
  CK(cudaMemcpy(&word, ctx->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (word != 0) {
    CK(cudaMemset(ctx->err, 0, sizeof(int)));
    return fail(ctx, word, word == DLM_ETIMEOUT ? "device wait timed out"
                                                : "device index check failed");
  }
  return DLM_OK;
}

int dlm_launches_per_step(const dlm_ctx* ctx) { return ctx ? ctx->launches : DLM_EINVAL; }

int dlm_test_exp2(const float* x, float* out, int n, void* stream) {
  g_create_error.clear();
  if (x == nullptr || out == nullptr || n < 0)
    return fail(nullptr, DLM_EINVAL, "test_exp2: NULL pointer or n < 0");
  if (n == 0) return DLM_OK;
  cudaError_t e = exp2_poly_apply(x, out, n, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(nullptr, "test_exp2 launch", e);
  return DLM_OK;
}

int dlm_test_withhold_loads(dlm_ctx* ctx, int n_launches) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (n_launches < 0) return fail(ctx, DLM_EINVAL, "n_launches must be >= 0");
  if (!ctx->bf16) return fail(ctx, DLM_EINVAL, "the fp32 model has no tensor-core GEMM");
  ctx->withhold_gemms = n_launches;
  return DLM_OK;
}

int dlm_set_stage_events(dlm_ctx* ctx, int stage, void* const* events, int n_pairs) {
  if (ctx == nullptr) return DLM_EINVAL;
  ctx->msg.clear();
  if (stage < 0 || stage >= DLM_NUM_STAGES || n_pairs < 0 || (n_pairs > 0 && events == nullptr))
    return fail(ctx, DLM_EINVAL, "bad stage or event array");
  ctx->ev.clear();
  ctx->ev_stage = n_pairs > 0 ? stage : -1;
  for (int i = 0; i < 2 * n_pairs; ++i) ctx->ev.push_back((cudaEvent_t)events[i]);
  ctx->ev_step = 0;
  return DLM_OK;
}

const char* dlm_last_error(const dlm_ctx* ctx) {
  return ctx ? ctx->msg.c_str() : g_create_error.c_str();
}

int dlm_trace_layout(int* kinds, int* ctas, int* slots) {
  if (kinds == nullptr || ctas == nullptr || slots == nullptr)
    return fail(nullptr, DLM_EINVAL, "trace_layout: NULL pointer argument");
  *kinds = kTraceKinds;
  *ctas = kTraceCtas;
  *slots = kTraceSlots;
#ifdef DLM_TRACE
  return DLM_OK;
#else
  return fail(nullptr, DLM_ESTATE, "trace: the library was built without DLM_TRACE");
#endif
}

int dlm_trace_read(unsigned long long* table, size_t words) {
  const size_t n = (size_t)kTraceKinds * kTraceCtas * kTraceSlots;
  if (table == nullptr || words < n)
    return fail(nullptr, DLM_EINVAL, "trace_read: table NULL or smaller than the layout");
#ifdef DLM_TRACE
  if (cudaError_t e = cudaDeviceSynchronize(); e != cudaSuccess)
    return cuda_fail(nullptr, "trace_read", e);
  // the tables of the translation units hold disjoint kinds: merge by max
  std::vector<unsigned long long> part(n);
  std::fill(table, table + n, 0ull);
  cudaError_t (*copies[])(unsigned long long*) = {trace_copy_gemm, trace_copy_simt, trace_copy_attn,
                                                  trace_copy_misc, trace_copy_sel};
  for (auto copy : copies) {
    if (cudaError_t e = copy(part.data()); e != cudaSuccess)
      return cuda_fail(nullptr, "trace_read", e);
    for (size_t i = 0; i < n; ++i) table[i] = std::max(table[i], part[i]);
  }
  return DLM_OK;
#else
  return fail(nullptr, DLM_ESTATE, "trace: the library was built without DLM_TRACE");
#endif
}

int dlm_trace_clear(void) {
#ifdef DLM_TRACE
  cudaError_t (*clears[])() = {trace_clear_gemm, trace_clear_simt, trace_clear_attn,
                               trace_clear_misc, trace_clear_sel};
  for (auto clear : clears)
    if (cudaError_t e = clear(); e != cudaSuccess) return cuda_fail(nullptr, "trace_clear", e);
  if (cudaError_t e = cudaDeviceSynchronize(); e != cudaSuccess)
    return cuda_fail(nullptr, "trace_clear", e);
  return DLM_OK;
#else
  return fail(nullptr, DLM_ESTATE, "trace: the library was built without DLM_TRACE");
#endif
}

}  // extern "C"

// ---------------------------------------------------------------------------
// attention without allocation: split partials in a fixed device array
// ---------------------------------------------------------------------------

// Row slots of split partials (one slot = one query row of one split of one
// (sequence, KV head)): 16384 slots = 8 MiB of partial outputs (128 floats
// each) + 128 KiB of (max, sum) pairs, plus one device error word.
constexpr int kNoAllocSlots = 16384;
constexpr int kNoAllocDh = 128;
static __device__ __align__(256) float g_noalloc_opart[(size_t)kNoAllocSlots * kNoAllocDh];
static __device__ __align__(256) float2 g_noalloc_ml[kNoAllocSlots];
static __device__ __align__(256) int g_noalloc_err[1];

namespace {

// Device addresses of the arrays above, looked up once per device (host code
// must not pass the arrays' names to a kernel: those are host stand-ins).
struct NoAllocScratch {
  std::once_flag once;
  cudaError_t status = cudaErrorNotReady;
  const char* what = "";
  float* opart = nullptr;
  float2* ml = nullptr;
  int* err = nullptr;
  int num_sms = 0;
};
constexpr int kMaxDevices = 64;
NoAllocScratch g_noalloc[kMaxDevices];

// runs once per device, with that device current
void noalloc_setup(NoAllocScratch& sc, int dev) {
  void* p = nullptr;
  cudaError_t e;
  if ((e = cudaGetSymbolAddress(&p, g_noalloc_opart)) != cudaSuccess) {
    sc.status = e;
    sc.what = "cudaGetSymbolAddress(partials)";
    return;
  }
  sc.opart = static_cast<float*>(p);
  if ((e = cudaGetSymbolAddress(&p, g_noalloc_ml)) != cudaSuccess) {
    sc.status = e;
    sc.what = "cudaGetSymbolAddress(max/sum)";
    return;
  }
  sc.ml = static_cast<float2*>(p);
  if ((e = cudaGetSymbolAddress(&p, g_noalloc_err)) != cudaSuccess) {
    sc.status = e;
    sc.what = "cudaGetSymbolAddress(error word)";
    return;
  }
  sc.err = static_cast<int*>(p);
  if ((e = cudaDeviceGetAttribute(&sc.num_sms, cudaDevAttrMultiProcessorCount, dev)) !=
      cudaSuccess) {
    sc.status = e;
    sc.what = "cudaDeviceGetAttribute(multiprocessor count)";
    return;
  }
  sc.status = cudaSuccess;
}

// the current device's scratch in *out, set up on first use; a DLM status
int noalloc_scratch(NoAllocScratch** out) {
  *out = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(nullptr, "cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices)
    return fail(nullptr, DLM_EINVAL, "attention_noalloc: device index out of range");
  NoAllocScratch& sc = g_noalloc[dev];
  std::call_once(sc.once, noalloc_setup, std::ref(sc), dev);
  if (sc.status != cudaSuccess) return cuda_fail(nullptr, sc.what, sc.status);
  *out = &sc;
  return DLM_OK;
}

}  // namespace

extern "C" {

int dlm_attention_noalloc(const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* lens, int max_len, void* o, int batch, int canvas,
                          int n_heads, int n_kv_heads, int head_dim, int kv_batch,
                          int kv_capacity, void* stream) {
  g_create_error.clear();
  if (!q || !k_cache || !v_cache || !lens || !o)
    return fail(nullptr, DLM_EINVAL, "attention_noalloc: NULL pointer argument");
  if (head_dim != kNoAllocDh || n_heads <= 0 || n_kv_heads <= 0 || n_heads % n_kv_heads != 0)
    return fail(nullptr, DLM_EINVAL,
                "attention_noalloc: needs head_dim 128 and n_heads a multiple of n_kv_heads");
  if (batch < 1 || canvas < 1 || batch > kv_batch || max_len < 0 ||
      (long)max_len + canvas > kv_capacity)
    return fail(nullptr, DLM_EINVAL,
                "attention_noalloc: need 1 <= batch <= kv_batch and max_len + canvas <= "
                "kv_capacity");
  NoAllocScratch* sc = nullptr;
  if (int rc = noalloc_scratch(&sc)) return rc;
  // the split plan of dlm_denoise_step for these sizes, restricted to plans
  // whose partials fit the fixed array (one split needs none, so one exists)
  dlm_ctx plan_ctx;
  plan_ctx.md = ModelDims{0, n_heads, n_kv_heads, head_dim, 0, -1, -1, kv_capacity, 2};
  plan_ctx.num_sms = sc->num_sms;
  const AttnPlan ap = plan_attention(&plan_ctx, batch, canvas, nullptr, max_len, kNoAllocSlots);
  const long slots = (long)batch * n_kv_heads * ap.nsplit * ap.R;
  if (ap.nsplit > 1 && ap.cluster <= 1 && slots > kNoAllocSlots) {
    g_create_error = "attention_noalloc: the split plan needs " + std::to_string(slots) +
                     " partial row slots; the static array holds " +
                     std::to_string(kNoAllocSlots);
    return DLM_EINVAL;
  }
  CUtensorMap tmK, tmV;
  const uint64_t planes = (uint64_t)kv_batch * n_kv_heads;
  if (!map_kv(&tmK, const_cast<void*>(k_cache), planes, kv_capacity, head_dim) ||
      !map_kv(&tmV, const_cast<void*>(v_cache), planes, kv_capacity, head_dim))
    return fail(nullptr, DLM_ECUDA, "attention_noalloc: cuTensorMapEncodeTiled failed");
  cudaStream_t st = (cudaStream_t)stream;
  CUtensorMap tmQ;
  const bool has_q = map_q(&tmQ, const_cast<void*>(q), (uint64_t)batch * canvas, n_heads,
                           head_dim, (uint32_t)(n_heads / n_kv_heads));
  cudaError_t e = attention_bf16(plan_ctx.md, ap, tmK, tmV, has_q ? &tmQ : nullptr, q, o,
                                 sc->opart, sc->ml, lens, nullptr, nullptr, sc->err, st);
  if (e != cudaSuccess) return cuda_fail(nullptr, "attention_noalloc launch", e);
  return DLM_OK;
}

int dlm_attention_noalloc_check(void* stream) {
  g_create_error.clear();
  NoAllocScratch* sc = nullptr;
  if (int rc = noalloc_scratch(&sc)) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(nullptr, "cudaStreamSynchronize", e);
  int word = 0;
  if ((e = cudaMemcpy(&word, sc->err, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(nullptr, "read the no-alloc error word", e);
  if (word == 0) return DLM_OK;
  if ((e = cudaMemset(sc->err, 0, sizeof(int))) != cudaSuccess)
    return cuda_fail(nullptr, "clear the no-alloc error word", e);
  return fail(nullptr, word, word == DLM_ETIMEOUT ? "attention_noalloc: device wait timed out"
                                                  : "attention_noalloc: device index check failed");
}

}  // extern "C"
