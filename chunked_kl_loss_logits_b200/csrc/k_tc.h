// Host-side launcher of the tcgen05 pair-GEMM kernels (internal; not part of the
// C ABI). Kept apart from the other launchers so that this header and k_tc.cu
// hold everything the tensor-core kernels are built from.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ckl {

struct TcMaps {
  CUtensorMap a, b, c;  // operands A and B; c = epilogue store target (G or dW)
};
enum class TcKind : int { LSE = 0, GRAD = 1, DH = 2, DW = 3, TKMAX = 4, TKEMIT = 5 };
struct TcLaunch {
  TcKind kind;
  int M, N, n_kb;  // output rows, output cols, 64-wide blocks along the contraction
  int n_split;     // DH only: contraction splits (>= 1)
  int V;           // LSE / GRAD: number of valid vocabulary columns
  float2* part;    // LSE
  int part_ld;     // LSE: rows of one vocabulary tile's partials (= Tc)
  const int32_t* sid;  // LSE: sorted cached ids per row (Tc x K)
  const float* sp;     // LSE: their teacher probabilities
  float* xpart;        // LSE: per-tile partial cross term, same layout as part
  int K;
  int store_e;     // LSE: also store exp(z - ref) in bf16 through map c, with ref the
                   // row's reference tok[row].w (log2 units), or the tile's maximum when
                   // that lies more than kRefGap above it
  const float4* tok;  // LSE with store_e: per-row values, .w = the reference
  const float4* cst;  // GRAD; DH with Hs (row factors)
  uint16_t* G;        // GRAD
  int64_t ldG;        // GRAD
  float* dHp;         // DH
  // DH, stored-exp backward: the epilogue warps also write Hs = bf16(c_t Hc) (M x N,
  // c_t the row factor from cst) for the dW contraction, before their first tile
  const uint16_t* Hc;
  uint16_t* Hs;
  float* dW;          // DW
  int first;          // DW: overwrite instead of accumulate
  // teacher top-K cache: TKMAX writes each row's best (logit, id) per vocabulary
  // tile into `part` (id stored as float bits); TKEMIT appends every (logit, id)
  // at least as good as the row's threshold `theta` to the row's candidate list.
  const float2* theta;
  float2* cand;
  int* cand_cnt;
  int cand_cap;
  unsigned* status;
  int num_sms;
};
int tc_bn(TcKind k);  // output columns of one tile of a kind (all its accumulators)
cudaError_t launch_tc(const TcMaps& maps, const TcLaunch& p, cudaStream_t s);

}  // namespace ckl
