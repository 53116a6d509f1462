// Element-wise kernels around the GEMMs: RoPE table, embedding gather, the
// projection epilogues (split-K sum, rotary embedding, KV-cache write,
// residual), KV copy-in and canvas initialisation.
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "kernels.h"

namespace dlm {

DLM_TRACE_STORAGE(misc)

namespace {

// cos/sin of pos * theta^(-2j/Dh), evaluated in double precision (positions
// reach 32k+, where a float32 angle would already be off by ~1e-3 rad)
__global__ void rope_table_kernel(float2* table, int Lcap, int half, double theta) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)Lcap * half) return;
  const int pos = (int)(i / half), j = (int)(i % half);
  const double inv_freq = pow(theta, -2.0 * (double)j / (double)(2 * half));
  double s, c;
  sincos((double)pos * inv_freq, &s, &c);
  table[i] = make_float2((float)c, (float)s);
}

template <typename T>
__global__ void embed_kernel(const int32_t* __restrict__ tokens, const T* __restrict__ emb,
                             T* __restrict__ x, int rows, int C, int d, int V, int B,
                             const uint8_t* __restrict__ done, int* n_active, int* err) {
  DLM_TRACE_CTA(TRACE_EMBED);
  pdl_wait_then_release();
  if (threadIdx.x == 0) DLM_TRACE_MARK(2);
  // this row's done flag and token are loaded together (and with block 0's
  // loads of every canvas's flag for the active count)
  const int r = blockIdx.x;
  const bool row_ok = r < rows;
  const bool dn = row_ok && done != nullptr && done[r / C] != 0;
  int t = row_ok ? tokens[r] : 0;
  if (blockIdx.x == 0 && n_active != nullptr) {
    __shared__ int cnt;
    if (threadIdx.x == 0) cnt = 0;
    __syncthreads();
    int mine = 0;
    for (int b = threadIdx.x; b < B; b += blockDim.x) mine += (done == nullptr || !done[b]);
    atomicAdd(&cnt, mine);
    __syncthreads();
    if (threadIdx.x == 0) *n_active = cnt;
  }
  if (!row_ok || dn) return;
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) raise_error(err, DLM_EBOUNDS);
    t = 0;
  }
  const uint4* src = reinterpret_cast<const uint4*>(emb + (size_t)t * d);
  uint4* dst = reinterpret_cast<uint4*>(x + (size_t)r * d);
  const int n16 = d * (int)sizeof(T) / 16;
  for (int i = threadIdx.x; i < n16; i += blockDim.x) dst[i] = src[i];
}

// block (row, group of heads): one rotary pair (j, j + Dh/2) per thread.
// The direct predecessor is always the GEMM that writes `part`; the active
// count, done flags, cache lengths and the rotary table come from earlier
// kernels, which have completed once this kernel may start (every kernel of
// the chain lets its successor launch only after its own wait), so they are
// read before the wait (through L2: a line left in L1 by an earlier step
// would be stale) and only the partial sums after it.
template <typename T>
__global__ void __launch_bounds__(256)
    qkv_epilogue_kernel(ModelDims md, const float* __restrict__ part, int splits, int rows, int C,
                        int seq_fixed, int head0, const int32_t* __restrict__ lens,
                        const float2* __restrict__ rope, T* __restrict__ q, T* __restrict__ kc,
                        T* __restrict__ vc, const uint8_t* __restrict__ done, const int* n_active,
                        int* err) {
  DLM_TRACE_CTA(seq_fixed < 0 ? TRACE_QKV_EPILOGUE : -1);
  const int r = blockIdx.x;
  const int half = md.Dh / 2;
  int seq, p_in;
  if (seq_fixed >= 0) {
    seq = seq_fixed;
    p_in = r;
  } else {
    seq = r / C;
    p_in = r - seq * C;
  }
  // issued together: active count, done flag, cache length
  const int na = n_active != nullptr ? __ldcg(n_active) : 1;
  const bool dn = seq_fixed < 0 && done != nullptr && __ldcg(done + seq) != 0;
  const int len = __ldcg(lens + seq);
  const int nheads = md.H + 2 * md.Hkv - head0;
  const int ncols = nheads * md.Dh;
  const int per_block = blockDim.x / half;
  const int item = blockIdx.y * per_block * half + threadIdx.x;
  bool active = na != 0 && !dn && item < nheads * half;
  const int hl = item / half, j = item - hl * half;
  const int hh = hl + head0;
  const int pos = len + p_in;
  const bool rotate = rope != nullptr && hh < md.H + md.Hkv;
  float2 cs = make_float2(1.f, 0.f);
  if (active && !DLM_IN_BOUNDS(pos, md.Lcap, err)) active = false;
  if (active && rotate) cs = rope[(size_t)pos * half + j];
  pdl_wait_then_release();
  if (threadIdx.x == 0) DLM_TRACE_MARK(2);
  if (!active) return;
  {
    const int cb = hl * md.Dh;
    float a = 0.f, b = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float* pr = part + ((size_t)s * rows + r) * ncols + cb;
      a += pr[j];
      b += pr[j + half];
    }
    if (rotate) {
      const float a2 = a * cs.x - b * cs.y;
      const float b2 = b * cs.x + a * cs.y;
      a = a2;
      b = b2;
    }
    T* dst;
    if (hh < md.H) {
      dst = q + ((size_t)r * md.H + hh) * md.Dh;
    } else if (hh < md.H + md.Hkv) {
      dst = kc + (((size_t)seq * md.Hkv + (hh - md.H)) * md.Lcap + pos) * md.Dh;
    } else {
      dst = vc + (((size_t)seq * md.Hkv + (hh - md.H - md.Hkv)) * md.Lcap + pos) * md.Dh;
    }
    dst[j] = from_f32<T>(a);
    dst[j + half] = from_f32<T>(b);
  }
}

// The direct predecessor is the GEMM that writes `part`; the active count,
// done flags and x come from earlier kernels (complete once this kernel may
// start) and are read before the wait, through L2.
template <typename T>
__global__ void wo_epilogue_kernel(const float* __restrict__ part, int splits, int rows, int d,
                                   int C, const T* __restrict__ x, T* __restrict__ y,
                                   const uint8_t* __restrict__ done, const int* n_active) {
  DLM_TRACE_CTA(TRACE_WO_EPILOGUE);
  const int r = blockIdx.y;
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const size_t i = (size_t)r * d + c;
  const int na = n_active != nullptr ? __ldcg(n_active) : 1;
  const bool dn = done != nullptr && __ldcg(done + r / C) != 0;
  const float xv = c < d ? to_f32(__ldcg(x + i)) : 0.f;
  pdl_wait_then_release();
  if (threadIdx.x == 0) DLM_TRACE_MARK(2);
  if (na == 0 || dn || c >= d) return;
  float acc = 0.f;
  for (int s = 0; s < splits; ++s) acc += part[((size_t)s * rows + r) * d + c];
  y[i] = from_f32<T>(xv + acc);
}

template <typename T>
__global__ void kv_copy_kernel(int Hkv, int Lcap, int Dh, int seq, int n,
                               const T* __restrict__ k, const T* __restrict__ v,
                               const int32_t* __restrict__ lens, T* kc, T* vc, int* err) {
  const int g = blockIdx.x, j = blockIdx.y;
  const int pos = lens[seq] + j;
  if (!DLM_IN_BOUNDS(pos, Lcap, err)) return;
  const size_t src = ((size_t)g * n + j) * Dh;
  const size_t dst = (((size_t)seq * Hkv + g) * Lcap + pos) * Dh;
  for (int t = threadIdx.x; t < Dh; t += blockDim.x) {
    kc[dst + t] = k[src + t];
    vc[dst + t] = v[src + t];
  }
}

__global__ void add_len_kernel(int32_t* lens, int seq, int n) { lens[seq] += n; }

__global__ void add_len_all_kernel(int32_t* lens, int B, int n) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) lens[b] += n;
}

// e4m3 quantisation of bf16 rows: s = max|x| / 448 (1 for an all-zero row),
// q = e4m3(x / s), round to nearest even, saturating.  One CTA per row;
// rows of finished canvases (row / C) are skipped.
__global__ void __launch_bounds__(256) quantize_rows_kernel(
    const __nv_bfloat16* __restrict__ x, int rows, int cols, uint8_t* __restrict__ q,
    float* __restrict__ scale, int C, const uint8_t* __restrict__ done, const int* n_active) {
  DLM_TRACE_CTA(TRACE_QUANTIZE);
  pdl_wait_then_release();
  if (threadIdx.x == 0) DLM_TRACE_MARK(2);
  if (n_active != nullptr && *n_active == 0) return;
  const int r = blockIdx.x;
  if (r >= rows || (done != nullptr && done[r / C])) return;
  const __nv_bfloat16* xr = x + (size_t)r * cols;
  float amax = 0.f;
  for (int i = threadIdx.x * 8; i < cols; i += blockDim.x * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(xr + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[u]));
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  __shared__ float wmax[8];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = wmax[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) amax = fmaxf(amax, wmax[w]);
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint8_t* qr = q + (size_t)r * cols;
  for (int i = threadIdx.x * 8; i < cols; i += blockDim.x * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(xr + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[u]));
      const uint32_t lo = __nv_cvt_float_to_fp8(__fdiv_rn(f.x, s), __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float_to_fp8(__fdiv_rn(f.y, s), __NV_SATFINITE, __NV_E4M3);
      packed[u >> 1] |= (lo | (hi << 8)) << (16 * (u & 1));
    }
    *reinterpret_cast<uint2*>(qr + i) = make_uint2(packed[0], packed[1]);
  }
  if (threadIdx.x == 0) scale[r] = s;
}

// NVFP4 rows (bf16 input, cols % 64 == 0): a float32 scale per row,
// s_r = amax(row) / (448 * 6) (1 for a zero row); per 16-element block an e4m3
// scale e4m3(amax(block) / (6 s_r)); elements e2m1(x / (sb * s_r)), 0 in a
// block whose scale is 0; every division and product in float32, round to
// nearest even, saturating.  Elements are packed two per byte, element 2i
// in the low nibble.  Block scales go to the layout the block-scaled tensor
// core reads after a 32-row x 16-byte copy replicated to all four lane
// quadrants: per 128-row block and 64-element k group one 512-byte chunk,
// byte (m % 32) * 16 + (m / 32) * 4 + s for row m of the row block and the
// s-th 16-element block of the k group.  One CTA per row, one thread per
// block (strided).  Rows of finished canvases (row / C, when done is given)
// are skipped.
__global__ void __launch_bounds__(256) quantize_rows_nvfp4_kernel(
    const __nv_bfloat16* __restrict__ x, int rows, int cols, uint8_t* __restrict__ q,
    uint8_t* __restrict__ sf, float* __restrict__ row_scale, int C,
    const uint8_t* __restrict__ done, const int* n_active) {
  DLM_TRACE_CTA(TRACE_QUANTIZE);
  pdl_wait_then_release();
  if (threadIdx.x == 0) DLM_TRACE_MARK(2);
  if (n_active != nullptr && *n_active == 0) return;
  const int r = blockIdx.x;
  if (r >= rows || (done != nullptr && done[r / C])) return;
  const __nv_bfloat16* xr = x + (size_t)r * cols;
  float amax = 0.f;
  for (int i = threadIdx.x * 8; i < cols; i += blockDim.x * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(xr + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[u]));
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  __shared__ float wmax[8];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = wmax[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) amax = fmaxf(amax, wmax[w]);
  const float sr = amax > 0.f ? __fdiv_rn(amax, 2688.f) : 1.f;   // 448 * 6
  const float six_sr = __fmul_rn(6.f, sr);
  const int kg = cols / 64;
  const int rb = r >> 7, m = r & 127;
  uint8_t* qr = q + (size_t)r * (cols / 2);
  for (int j = threadIdx.x; j < cols / 16; j += blockDim.x) {
    float f[16];
    const uint4* src = reinterpret_cast<const uint4*>(xr + j * 16);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 v = src[h];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[u]));
        f[8 * h + 2 * u] = t.x;
        f[8 * h + 2 * u + 1] = t.y;
      }
    }
    float ab = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) ab = fmaxf(ab, fabsf(f[e]));
    const __nv_fp8_storage_t sbq = __nv_cvt_float_to_fp8(__fdiv_rn(ab, six_sr), __NV_SATFINITE,
                                                         __NV_E4M3);
    const float sbv = __half2float(__half(__nv_cvt_fp8_to_halfraw(sbq, __NV_E4M3)));
    const float scale = __fmul_rn(sbv, sr);
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float ratio = scale > 0.f ? __fdiv_rn(f[e], scale) : 0.f;
      const uint32_t code =
          (uint32_t)__nv_cvt_float_to_fp4(ratio, __NV_E2M1, cudaRoundNearest) & 0xFu;
      packed[e >> 3] |= code << (4 * (e & 7));
    }
    *reinterpret_cast<uint2*>(qr + j * 8) = make_uint2(packed[0], packed[1]);
    const int g = j >> 2, sblk = j & 3;
    sf[((size_t)rb * kg + g) * 512 + (m & 31) * 16 + (m >> 5) * 4 + sblk] = sbq;
  }
  if (threadIdx.x == 0) row_scale[r] = sr;
}

// test hook: the attention's polynomial exp2 on given arguments
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = exp2_poly(x[i]);
}

__global__ void canvas_init_kernel(int C, int V, int mask_id, int uniform, uint32_t s0,
                                   uint32_t s1, int32_t* tokens, uint8_t* committed,
                                   int32_t* step, uint8_t* done, int32_t* eos_pos,
                                   int32_t* prev_cand, int32_t* stable) {
  const int b = blockIdx.x;
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    if (prev_cand != nullptr) prev_cand[(size_t)b * C + i] = -1;
    int32_t t = mask_id;
    if (uniform) {
      const U32x4 w = philox10(U32x4{(uint32_t)b, 0u, (uint32_t)i, kRenoiseWord}, s0, s1);
      t = uniform_id(w.a, V);
    }
    tokens[(size_t)b * C + i] = t;
    committed[(size_t)b * C + i] = 0;
  }
  if (threadIdx.x == 0) {
    step[b] = 0;
    done[b] = 0;
    eos_pos[b] = -1;
    if (stable != nullptr) stable[b] = 0;
  }
}

}  // namespace

cudaError_t rope_table_init(float2* table, int Lcap, int Dh, double theta, cudaStream_t st) {
  const int64_t n = (int64_t)Lcap * (Dh / 2);
  rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(table, Lcap, Dh / 2, theta);
  return cudaGetLastError();
}

cudaError_t embed_rows(const ModelDims& md, const int32_t* tokens, const void* emb, void* x,
                       int rows, int C, int B, const uint8_t* done, int* n_active, int* err,
                       cudaStream_t st) {
  if (md.esize == 2)
    return launch_pdl(embed_kernel<__nv_bfloat16>, dim3(rows), dim3(128), 0, st, tokens,
                      (const __nv_bfloat16*)emb, (__nv_bfloat16*)x, rows, C, md.d, md.V, B, done,
                      n_active, err);
  return launch_pdl(embed_kernel<float>, dim3(rows), dim3(128), 0, st, tokens, (const float*)emb,
                    (float*)x, rows, C, md.d, md.V, B, done, n_active, err);
}

cudaError_t qkv_epilogue(const ModelDims& md, const float* part, int splits, int rows, int C,
                         int seq_fixed, int head0, const int32_t* lens, const float2* rope,
                         void* q, void* kcache, void* vcache, const uint8_t* done,
                         const int* n_active, int* err, cudaStream_t st) {
  const int half = md.Dh / 2;
  const int per_block = 256 / half;   // heads per block
  dim3 grid(rows, (md.H + 2 * md.Hkv - head0 + per_block - 1) / per_block);
  if (md.esize == 2)
    return launch_pdl(qkv_epilogue_kernel<__nv_bfloat16>, grid, dim3(per_block * half), 0, st, md, part,
                      splits, rows, C, seq_fixed, head0, lens, rope, (__nv_bfloat16*)q,
                      (__nv_bfloat16*)kcache, (__nv_bfloat16*)vcache, done, n_active, err);
  return launch_pdl(qkv_epilogue_kernel<float>, grid, dim3(per_block * half), 0, st, md, part, splits,
                    rows, C, seq_fixed, head0, lens, rope, (float*)q, (float*)kcache,
                    (float*)vcache, done, n_active, err);
}

cudaError_t wo_epilogue(const ModelDims& md, const float* part, int splits, int rows, int C,
                        const void* x, void* y, const uint8_t* done, const int* n_active,
                        cudaStream_t st) {
  dim3 grid((md.d + 255) / 256, rows);
  if (md.esize == 2)
    return launch_pdl(wo_epilogue_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, part, splits,
                      rows, md.d, C, (const __nv_bfloat16*)x, (__nv_bfloat16*)y, done, n_active);
  return launch_pdl(wo_epilogue_kernel<float>, grid, dim3(256), 0, st, part, splits, rows, md.d,
                    C, (const float*)x, (float*)y, done, n_active);
}

cudaError_t kv_copy_in(const ModelDims& md, int seq, int n, const void* k, const void* v,
                       const int32_t* lens, void* kcache, void* vcache, int* err,
                       cudaStream_t st) {
  dim3 grid(md.Hkv, n);
  const int threads = md.Dh < 128 ? md.Dh : 128;
  if (md.esize == 2)
    kv_copy_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(
        md.Hkv, md.Lcap, md.Dh, seq, n, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, lens,
        (__nv_bfloat16*)kcache, (__nv_bfloat16*)vcache, err);
  else
    kv_copy_kernel<float><<<grid, threads, 0, st>>>(md.Hkv, md.Lcap, md.Dh, seq, n,
                                                    (const float*)k, (const float*)v, lens,
                                                    (float*)kcache, (float*)vcache, err);
  return cudaGetLastError();
}

cudaError_t add_len(int32_t* lens, int seq, int n, cudaStream_t st) {
  add_len_kernel<<<1, 1, 0, st>>>(lens, seq, n);
  return cudaGetLastError();
}

cudaError_t canvas_init(const ModelDims& md, int B, int C, int corruption, uint64_t seed,
                        int32_t* tokens, uint8_t* committed, int32_t* step, uint8_t* done,
                        int32_t* eos_pos, int32_t* prev_cand, int32_t* stable, cudaStream_t st) {
  const int threads = C < 1024 ? ((C + 31) / 32) * 32 : 1024;
  canvas_init_kernel<<<B, threads, 0, st>>>(C, md.V, md.mask_id, corruption == DLM_UNIFORM,
                                            (uint32_t)(seed & 0xFFFFFFFFull),
                                            (uint32_t)(seed >> 32), tokens, committed, step,
                                            done, eos_pos, prev_cand, stable);
  return cudaGetLastError();
}

cudaError_t quantize_rows_e4m3(const void* x, int rows, int cols, uint8_t* q, float* scale, int C,
                               const uint8_t* done, const int* n_active, cudaStream_t st) {
  if (cols % 8 != 0) return cudaErrorInvalidValue;
  return launch_pdl(quantize_rows_kernel, dim3(rows), dim3(256), 0, st,
                    (const __nv_bfloat16*)x, rows, cols, q, scale, C, done, n_active);
}

cudaError_t quantize_rows_nvfp4(const void* x, int rows, int cols, uint8_t* q, uint8_t* sf,
                                float* row_scale, int C, const uint8_t* done, const int* n_active,
                                cudaStream_t st) {
  if (cols % 64 != 0) return cudaErrorInvalidValue;
  return launch_pdl(quantize_rows_nvfp4_kernel, dim3(rows), dim3(256), 0, st,
                    (const __nv_bfloat16*)x, rows, cols, q, sf, row_scale, C, done, n_active);
}

cudaError_t exp2_poly_apply(const float* x, float* out, int n, cudaStream_t st) {
  exp2_poly_kernel<<<(n + 255) / 256, 256, 0, st>>>(x, out, n);
  return cudaGetLastError();
}

cudaError_t add_len_all(int32_t* lens, int B, int n, cudaStream_t st) {
  add_len_all_kernel<<<(B + 127) / 128, 128, 0, st>>>(lens, B, n);
  return cudaGetLastError();
}

}  // namespace dlm
