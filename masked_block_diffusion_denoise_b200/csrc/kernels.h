// Host-side launchers of the library's kernels (one per .cu file section).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lm_epilogue.cuh"

namespace dlm {

// GEMM epilogues: f32 (split-K) partials; the LM head's vocabulary
// reduction; the QKV projection with RoPE and q / KV-cache stores; the output
// projection with the residual add.  The last two run when K is not split.
enum { EPI_F32 = 0, EPI_LM = 1, EPI_QKV = 2, EPI_RESID = 3 };

struct GemmPlan {
  int M, N, K;
  int BN;       // 128 or 256 (tcgen05); 64 (fp32 SIMT)
  int splits;   // K splits (EPI_F32 only)
  int epi;      // EPI_F32 / EPI_LM
  int f8 = 0;       // e4m3 operands (tcgen05 only; EPI_LM and EPI_F32)
  int f4 = 0;       // NVFP4 operands with block scales (tcgen05, BN 128; EPI_LM, EPI_F32)
};

struct ModelDims;

// destinations of the fused projection epilogues (bf16 model)
struct ProjEpi {
  int H = 0, Hkv = 0, Dh = 0, Lcap = 0, C = 1;
  const int32_t* lens = nullptr;     // [B] prefix lengths (canvas slots follow)
  const float2* rope = nullptr;      // [Lcap][Dh/2] cos/sin, or null
  void* q = nullptr;                 // EPI_QKV: [M][H][Dh]
  void* kcache = nullptr;            // EPI_QKV: [B][Hkv][Lcap][Dh]
  void* vcache = nullptr;
  const void* x = nullptr;           // EPI_RESID: residual [M][N]
  void* y = nullptr;                 // EPI_RESID: [M][N]
};

// Device timeline (DLM_TRACE builds): one kind per kernel of the step
enum TraceKind {
  TRACE_EMBED = 0,
  TRACE_QKV_GEMM = 1,
  TRACE_QKV_EPILOGUE = 2,
  TRACE_ATTENTION = 3,
  TRACE_ATTN_COMBINE = 4,
  TRACE_WO_GEMM = 5,
  TRACE_WO_EPILOGUE = 6,
  TRACE_QUANTIZE = 7,
  TRACE_LM_HEAD = 8,
  TRACE_COMMIT = 9,
  TRACE_KINDS_USED = 10
};
#ifdef DLM_TRACE
// each translation unit's table (see DLM_TRACE_STORAGE)
cudaError_t trace_copy_gemm(unsigned long long* host);
cudaError_t trace_clear_gemm();
cudaError_t trace_copy_simt(unsigned long long* host);
cudaError_t trace_clear_simt();
cudaError_t trace_copy_attn(unsigned long long* host);
cudaError_t trace_clear_attn();
cudaError_t trace_copy_misc(unsigned long long* host);
cudaError_t trace_clear_misc();
cudaError_t trace_copy_sel(unsigned long long* host);
cudaError_t trace_clear_sel();
#endif

struct GemmIO {
  float* out = nullptr;        // EPI_F32: [splits][M][N]
  float* part = nullptr;       // EPI_LM:  [M][kLmFields][n_part]
  LmEpi epi{};
  ProjEpi proj{};
  const uint8_t* done = nullptr;
  const int* n_active = nullptr;
  int* err = nullptr;
  int trace_kind = -1;         // TraceKind of this launch, -1: not traced
  int withhold_loads = 0;      // failure-detection test: see dlm_test_withhold_loads
  const uint8_t* sfa = nullptr;   // NVFP4: block scales of A and B ([128-row block][K/64][512])
  const uint8_t* sfb = nullptr;
};

// ---- gemm_tc.cu: bf16 tcgen05 GEMM ---------------------------------------
cudaError_t gemm_tc(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmPlan& plan,
                    const GemmIO& io, int num_sms, cudaStream_t st);
int gemm_tc_smem_bytes(int BN);
// rows of the A (activation) box: all rows in use, rounded up to 8, at most 128
int gemm_tc_a_rows(int M);
// LM partials per row written by the EPI_LM launch of `plan` (one per CTA slot)
int gemm_tc_lm_partials(const GemmPlan& plan, int num_sms);

// ---- gemm_simt.cu: fp32 GEMM on the CUDA cores (fp32 model) ----------------
cudaError_t gemm_f32(const float* A, const float* B, const GemmPlan& plan, const GemmIO& io,
                     cudaStream_t st);

// ---- misc.cu: embedding, projection epilogues, cache writes, canvas init --
struct ModelDims {
  int d, H, Hkv, Dh, V, mask_id, eos_id;
  int Lcap;      // KV slots per (sequence, KV head)
  int esize;     // element bytes
};

cudaError_t rope_table_init(float2* table, int Lcap, int Dh, double theta, cudaStream_t st);

// x[r] = E[tokens[r]] for r < rows; skips rows of finished canvases; block 0
// also writes *n_active = number of unfinished canvases (done may be null)
cudaError_t embed_rows(const ModelDims& md, const int32_t* tokens, const void* emb, void* x,
                       int rows, int C, int B, const uint8_t* done, int* n_active, int* err,
                       cudaStream_t st);

// Sum split-K partials of the fused QKV projection, rotate q and k, store q
// ([rows][H][Dh]) and k, v into the cache at slot lens[seq] + position.
// Row r is (seq = r / C, position = r % C) or, with seq_fixed >= 0, (seq_fixed,
// position = r).  head0 = first head of the partial columns (0: q, k, v;
// H: k, v only).
cudaError_t qkv_epilogue(const ModelDims& md, const float* part, int splits, int rows, int C,
                         int seq_fixed, int head0, const int32_t* lens, const float2* rope,
                         void* q, void* kcache, void* vcache, const uint8_t* done,
                         const int* n_active, int* err, cudaStream_t st);

// y = x + sum of split-K partials of o W_o^T
cudaError_t wo_epilogue(const ModelDims& md, const float* part, int splits, int rows, int C,
                        const void* x, void* y, const uint8_t* done, const int* n_active,
                        cudaStream_t st);

// copy caller K/V [Hkv][n][Dh] into the cache of `seq` at slots lens[seq]..
cudaError_t kv_copy_in(const ModelDims& md, int seq, int n, const void* k, const void* v,
                       const int32_t* lens, void* kcache, void* vcache, int* err,
                       cudaStream_t st);

cudaError_t add_len(int32_t* lens, int seq, int n, cudaStream_t st);

cudaError_t canvas_init(const ModelDims& md, int B, int C, int corruption, uint64_t seed,
                        int32_t* tokens, uint8_t* committed, int32_t* step, uint8_t* done,
                        int32_t* eos_pos, int32_t* prev_cand, int32_t* stable, cudaStream_t st);

// lens[b] += n for b < B
cudaError_t add_len_all(int32_t* lens, int B, int n, cudaStream_t st);

// e4m3 rows with one float32 scale each (bf16 input, cols % 8 == 0); rows of
// finished canvases (row / C, when done is given) are skipped
cudaError_t quantize_rows_e4m3(const void* x, int rows, int cols, uint8_t* q, float* scale, int C,
                               const uint8_t* done, const int* n_active, cudaStream_t st);

// NVFP4 rows (bf16 input, cols % 64 == 0): packed e2m1 elements q [rows][cols/2]
// (element 2i in the low nibble), e4m3 block scales of 16 in the block-scaled
// MMA's layout sf [ceil(rows/128)][cols/64][512] (see the kernel), a float32
// scale per row; rows of finished canvases are skipped
cudaError_t quantize_rows_nvfp4(const void* x, int rows, int cols, uint8_t* q, uint8_t* sf,
                                float* row_scale, int C, const uint8_t* done, const int* n_active,
                                cudaStream_t st);

// out[i] = exp2_poly(x[i]) (the attention's exponential on the FMA pipe)
cudaError_t exp2_poly_apply(const float* x, float* out, int n, cudaStream_t st);

// ---- attention.cu ------------------------------------------------------------
struct AttnPlan {
  int B, C, G, R, rtiles;   // G = H / Hkv, R = G * C query rows per (seq, kv head)
  int chunk, nsplit;        // keys per split (multiple of 128), splits per (seq, kv head)
  int cluster = 1;          // nsplit (<= 16) when the splits combine inside a cluster
  int rows = 128;           // query rows per CTA
};

// clusters of n (2..16) attention CTAs that fit on the device at once (0: none)
int attn_cluster_capacity(int n);

// bf16: tcgen05 flash attention over [prefix ; canvas] keys (S and O in tensor
// memory, K/V by TMA), split over keys; up to 16 splits combine inside a
// thread-block cluster, more write partials for the combine kernel.
// tmQ: q [positions][H][Dh] as a 3-D map with box (64, G, 128/G), used when G
// divides 128 (else, or when null, the query tile is loaded with plain loads)
cudaError_t attention_bf16(const ModelDims& md, const AttnPlan& ap, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const CUtensorMap* tmQ, const void* q, void* o,
                           float* opart, float2* ml, const int32_t* lens, const uint8_t* done,
                           const int* n_active, int* err, cudaStream_t st);
// fp32: one thread per query row
cudaError_t attention_f32(const ModelDims& md, int B, int C, const float* q, const float* kcache,
                          const float* vcache, float* o, const int32_t* lens,
                          const uint8_t* done, const int* n_active, int* err,
                          cudaStream_t st);

// ---- select.cu ------------------------------------------------------------------
struct SelectArgs {
  int B, C, S, V;
  int quota;             // effective quota (>= 1)
  float threshold;
  int eb;                // entropy-bound rule
  float bound;
  int uniform;           // re-noise with uniform ids
  int mask_id, eos_id;
  uint32_t seed_lo, seed_hi;
  int stability_steps;   // adaptive stopping (stop_entropy > 0)
  float stop_entropy;
  int editing;           // token editing of committed positions
  float edit_thr;
};

// Kernel (c).  With `part` != null it first combines the LM partials of each
// row of its canvas (n_part per row) into cand / conf / ent (written to those
// buffers), then selects from them; with part == null it selects from the
// given cand / conf / ent.
cudaError_t commit_step(const SelectArgs& a, int32_t* tokens, uint8_t* committed, int32_t* step,
                        uint8_t* done, int32_t* eos_pos, int32_t* prev_cand, int32_t* stable,
                        const float* part, int n_part, int32_t* cand, float* conf, float* ent,
                        dlm_canvas_stats* stats, const int* n_active, int* err, cudaStream_t st);

}  // namespace dlm
