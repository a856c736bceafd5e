// True-fp32 path (FFMA on the CUDA cores) for float32 inputs: the tensor cores
// offer only tf32 for 32-bit operands, which cannot hold the fp32 accuracy of the
// loss. One 64x64 output tile per block, 4x4 outputs per thread, three
// epilogues: the per-tile (max, sum of exp) of the logits, the scaled gradient
// of the logits, and a plain store / accumulate for the dH and dW products.
#include "common.cuh"
#include "kernels.h"

namespace ckl {

namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;
constexpr float kLog2e = 1.4426950408889634f;

struct EpiLse {  // part[tile_col][row] = (max, sum exp2) over the tile's valid columns
  float2* part;
  int ld;
};
struct EpiGrad {  // G[row][col] = gmul_row * exp(z - lse_row)
  const float4* cst;
  float* G;
  int64_t ldG;
};
struct EpiStore {  // C[row][col] (+)= acc
  float* C;
  int64_t ldc;
  int beta;
};

__device__ __forceinline__ float half_warp_max(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float half_warp_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void epilogue(const EpiLse& e, int r0, int c0, float (&acc)[4][4], int M,
                                         int N) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float x[4];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[j] = (c0 + j < N) ? acc[i][j] * kLog2e : -INFINITY;
      mx = fmaxf(mx, x[j]);
    }
    mx = half_warp_max(mx);
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) s += (c0 + j < N) ? ex2_approx(x[j] - mx) : 0.f;
    s = half_warp_sum(s);
    if ((threadIdx.x & 15) == 0 && r0 + i < M)
      e.part[(int64_t)blockIdx.x * e.ld + r0 + i] = make_float2(mx, s);
  }
}

__device__ __forceinline__ void epilogue(const EpiGrad& e, int r0, int c0, float (&acc)[4][4],
                                         int M, int N) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (r0 + i >= M) continue;
    const float4 c = e.cst[r0 + i];
    const float lse2 = c.x * kLog2e;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (c0 + j < N)
        e.G[(int64_t)(r0 + i) * e.ldG + c0 + j] = c.y * ex2_approx(fmaf(acc[i][j], kLog2e, -lse2));
  }
}

__device__ __forceinline__ void epilogue(const EpiStore& e, int r0, int c0, float (&acc)[4][4],
                                         int M, int N) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (r0 + i >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (c0 + j >= N) continue;
      float* p = e.C + (int64_t)(r0 + i) * e.ldc + c0 + j;
      *p = e.beta ? *p + acc[i][j] : acc[i][j];
    }
  }
}

// out(m, n) = sum_k A[m*sam + k*sak] * B[n*sbn + k*sbk] over one 64x64 tile.
template <class Epi>
__global__ void __launch_bounds__(NT) simt_tile_kernel(const float* __restrict__ A, int64_t sam,
                                                        int64_t sak, const float* __restrict__ B,
                                                        int64_t sbn, int64_t sbk, int M, int N,
                                                        int Kd, Epi epi) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < Kd; k0 += BK) {
    for (int e = threadIdx.x; e < BM * BK; e += NT) {
      int mm, kk;
      if (sak == 1) { mm = e / BK; kk = e % BK; } else { mm = e % BM; kk = e / BM; }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < Kd) ? A[(int64_t)gm * sam + (int64_t)gk * sak] : 0.f;
    }
    for (int e = threadIdx.x; e < BN * BK; e += NT) {
      int nn, kk;
      if (sbk == 1) { nn = e / BK; kk = e % BK; } else { nn = e % BN; kk = e / BN; }
      const int gn = n0 + nn, gk = k0 + kk;
      Bs[kk][nn] = (gn < N && gk < Kd) ? B[(int64_t)gn * sbn + (int64_t)gk * sbk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  epilogue(epi, m0 + ty * 4, n0 + tx * 4, acc, M, N);
}

inline dim3 grid_for(int M, int N) { return dim3((N + BN - 1) / BN, (M + BM - 1) / BM); }

}  // namespace

void launch_simt_lse(const float* Hc, const float* W, int Tc, int V, int d, float2* part,
                     cudaStream_t s) {
  simt_tile_kernel<EpiLse><<<grid_for(Tc, V), NT, 0, s>>>(Hc, d, 1, W, d, 1, Tc, V, d,
                                                          EpiLse{part, Tc});
}

void launch_simt_grad(const float* Hc, const float* W, int Tc, int V, int d, const float4* cst,
                      float* G, int64_t ldG, cudaStream_t s) {
  simt_tile_kernel<EpiGrad><<<grid_for(Tc, V), NT, 0, s>>>(Hc, d, 1, W, d, 1, Tc, V, d,
                                                           EpiGrad{cst, G, ldG});
}

void launch_simt_gemm(const float* A, int64_t sam, int64_t sak, const float* B, int64_t sbn,
                      int64_t sbk, float* C, int64_t ldc, int M, int N, int Kd, int beta,
                      cudaStream_t s) {
  simt_tile_kernel<EpiStore><<<grid_for(M, N), NT, 0, s>>>(A, sam, sak, B, sbn, sbk, M, N, Kd,
                                                           EpiStore{C, ldc, beta});
}

}  // namespace ckl
