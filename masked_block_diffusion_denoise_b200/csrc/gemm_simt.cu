// fp32 GEMM on the CUDA cores for the float32 model: D[M][N] = A[M][K] .
// B[N][K]^T with 64x64 tiles, 4x4 outputs per thread, the same two
// epilogues as the tensor-core engine (f32 split-K partials, or the LM head's
// fused vocabulary reduction over 64-column tiles).
#include "kernels.h"

namespace dlm {

DLM_TRACE_STORAGE(simt)

namespace {

constexpr int kT = 64;
constexpr int kTK = 16;

struct SimtParams {
  int M, N, K, splits, n_tiles;
  float* out;
  float* part;   // EPI_LM partials, [M][kLmFields][n_tiles]
  LmEpi epi;
  const uint8_t* done;
  const int* n_active;
  int trace_kind;
};

template <int EPI>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A,
                                                       const float* __restrict__ B,
                                                       const SimtParams p) {
  DLM_TRACE_CTA(p.trace_kind);
  pdl_wait_then_release();
  if (threadIdx.x == 0) DLM_TRACE_MARK(2);
  if (p.n_active != nullptr && *p.n_active == 0) return;
  __shared__ float As[kTK][kT + 4];
  __shared__ float Bs[kTK][kT + 4];
  __shared__ float Ts[kT][kT + 1];
  const int m0 = blockIdx.y * kT, n0 = blockIdx.x * kT, split = blockIdx.z;
  const int kchunks = (p.K + kTK - 1) / kTK;
  const int kc0 = (int)((long long)split * kchunks / p.splits);
  const int kc1 = (int)((long long)(split + 1) * kchunks / p.splits);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int kc = kc0; kc < kc1; ++kc) {
    const int k0 = kc * kTK;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = threadIdx.x + i * 256;
      const int r = idx >> 4, kk = idx & 15;
      const int k = k0 + kk;
      As[kk][r] = (m0 + r < p.M && k < p.K) ? A[(size_t)(m0 + r) * p.K + k] : 0.f;
      Bs[kk][r] = (n0 + r < p.N && k < p.K) ? B[(size_t)(n0 + r) * p.K + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kTK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  if constexpr (EPI == EPI_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = m0 + ty * 4 + i;
      if (row >= p.M) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = n0 + tx * 4 + j;
        if (col < p.N) p.out[((size_t)split * p.M + row) * p.N + col] = acc[i][j];
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) Ts[ty * 4 + i][tx * 4 + j] = acc[i][j];
    __syncthreads();
    if (threadIdx.x < kT) {
      const int row = m0 + threadIdx.x;
      if (row < p.M) {
        const int canvas = row / p.epi.C;
        const int pos = row - canvas * p.epi.C;
        if (p.done == nullptr || p.done[canvas] == 0) {
          const int step = p.epi.step[canvas];
          const float inv_t = lm_inv_temp(p.epi, step);
          RowState rs;
          rs_init(rs);
#pragma unroll 1
          for (int c = 0; c < kT; c += 32) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = Ts[threadIdx.x][c + j];
            rs_update<32>(rs, v, n0 + c, inv_t, p.epi, canvas, pos, step);
          }
          rs_store(p.part, p.n_tiles, (size_t)row, blockIdx.x, rs);
        }
      }
    }
  }
}

}  // namespace

cudaError_t gemm_f32(const float* A, const float* B, const GemmPlan& plan, const GemmIO& io,
                     cudaStream_t st) {
  SimtParams p{};
  p.M = plan.M;
  p.N = plan.N;
  p.K = plan.K;
  p.splits = plan.splits;
  p.n_tiles = (plan.N + kT - 1) / kT;
  p.out = io.out;
  p.part = io.part;
  p.epi = io.epi;
  p.epi.n_tiles = p.n_tiles;
  p.done = io.done;
  p.n_active = io.n_active;
  p.trace_kind = io.trace_kind;
  dim3 grid(p.n_tiles, (plan.M + kT - 1) / kT, plan.epi == EPI_LM ? 1 : plan.splits);
  if (plan.epi == EPI_LM) return launch_pdl(gemm_f32_kernel<EPI_LM>, grid, dim3(256), 0, st, A, B, p);
  return launch_pdl(gemm_f32_kernel<EPI_F32>, grid, dim3(256), 0, st, A, B, p);
}

}  // namespace dlm
