// Host-side launchers of the library's kernels (internal; not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "k_tc.h"

namespace ckl {

// Per-token values of the chunk being processed, in the workspace.
//   tok[i] = (ent_i, cross_i, M_i, r2_i)   from the teacher kernel; r2 = the reference
//            logit of the stored-exp backward (log2 units; 0 when not used)
//   cst[i] = (lse_i, gmul_i, s_i, R_i)     from the combine: gmul = s * M, s = mask/N,
//            R = the row's reference of the stored exps (stored-exp backward only)
struct Misc;
struct ChunkBufs {
  float4* tok;
  float4* cst;
  float* zk;     // Tc x K student logits at the cached ids
  float* Pk;     // Tc x K total teacher probability of each slot's id; 0 on every slot
                 // but the first that holds a given id (so each id is corrected once)
  float2* part;  // n_vt x Tc partial (max, sum) of exp over one vocabulary tile, log2 units
  float* xpart;  // bf16: n_vt x Tc partial sum_k p_k z_k over the ids inside one vocabulary tile
  int32_t* sid;  // bf16: Tc x K cached ids of each token, ascending
  float* sp;     // bf16: Tc x K teacher probability of each sorted slot
  void* G;       // Tc x ldG scaled gradient of the logits (bf16 or f32)
  float* dHp;    // split-K partials of dH (bf16 path)
  int* rep;      // stored-exp backward: [count, rows...] of the rows to repair this chunk
  struct Misc* misc;
};

// Call-wide scalars in the workspace.
struct Misc {
  double N;         // number of unmasked tokens
  double loss_sum;  // sum of mask_t * l_t
  float invN;       // 1 / N, or 0 when N == 0
  float pad[3];
};

// ---- small kernels (k_small.cu)
void launch_mask_count(const uint8_t* mask, int64_t T, Misc* misc, cudaStream_t s);
// bf16: teacher softmax, merged P, entropy term and each token's ids sorted with
// their probabilities (the forward contraction picks the student logits there).
// Ids are checked against V_all and written relative to v0 (vocabulary split
// over ranks: this rank holds rows [v0, v0 + V_loc) of W; otherwise v0 = 0,
// V_all = V_loc). With Hc (the chunk's hidden states; W and d then too): also the
// reference logit r2 of the stored-exp backward into tok.w, and the chunk's
// repair list is emptied. behind: launched as a dependent of the kernel just
// enqueued on s (the previous chunk's dH contraction), which it may overlap; its
// completion still implies that kernel's.
void launch_teacher(const int32_t* idx, const float* logit, int64_t t0, int Tc, int V_all, int v0,
                    int V_loc, int K, const ChunkBufs& b, unsigned* status, const uint16_t* Hc,
                    const uint16_t* W, int d, bool behind, cudaStream_t s);
// fp32: as launch_teacher, plus the student logits at the ids by dot products.
template <typename Tin>
void launch_gather(const Tin* H, const Tin* W, const int32_t* idx, const float* logit, int64_t t0,
                   int Tc, int d, int V, int K, const ChunkBufs& b, unsigned* status,
                   cudaStream_t s);
// stats != nullptr: write this rank's per-token (max2, sum, cross, 0) and stop.
// row_ref (stored-exp backward): also each row's reference R into cst.w, rows whose
// tiles outgrew the teacher kernel's reference joining the repair list.
void launch_combine(int64_t t0, int Tc, int n_vt, const uint8_t* mask, const ChunkBufs& b,
                    float* lse_all, float* ell_all, float4* stats, bool row_ref, cudaStream_t s);
// Merge world x Tc gathered stats (rank-major) into lse, l_t and the multipliers
// (and, with row_ref, this rank's row references and repair list).
void launch_vp_merge(int64_t t0, int Tc, int world, int rank, const float4* stats_all,
                     const uint8_t* mask, const ChunkBufs& b, float* lse_all, float* ell_all,
                     bool row_ref, cudaStream_t s);
// G at the cached ids, in place: G -= s P_k where G is gmul exp(z - lse); with
// row_ref (G holds the stored exp(z - R)) G -= (P_k / M) exp(lse - R).
template <typename Tg>
// ldG: fp32 row stride of G; bf16: the number of 64-wide vocabulary blocks (G blocked).
void launch_fixup(const int32_t* idx, int64_t t0, int Tc, int K, int V, int v0, int64_t ldG,
                  const ChunkBufs& b, bool row_ref, cudaStream_t s);
// Stored-exp backward: rescale the rows on the chunk's repair list to their common
// reference R, in place (G blocked, bf16); nothing to do for an empty list.
void launch_repair(uint16_t* G, int Tc, int V, const ChunkBufs& b, int num_sms, cudaStream_t s);
// Sum of the n_split partials of dH_c -> bf16 dH. With cst (stored-exp backward)
// each row is multiplied by c_t = gmul exp(R - lse). Launched as a dependent of the
// kernel just enqueued on s (the chunk's dW contraction), which it overlaps on at
// most num_sms blocks; its completion still implies that kernel's.
void launch_dh_reduce_bf16(const float* dHp, int n_split, int64_t n_elem, uint16_t* dH, int d,
                           const float4* cst, int num_sms, cudaStream_t s);
// One thread waits on a barrier nothing arrives at until the wait bound fires.
void launch_wait_selftest(unsigned* status, long long* cycles, cudaStream_t s);
// Top-K cache with the vocabulary split over ranks: pack this rank's K best as
// (logit, global id); regroup the gathered pairs per row for the final select.
void launch_topk_pack(const int32_t* idx, const float* lg, int64_t n, int v0, float2* out,
                      cudaStream_t s);
void launch_topk_regroup(const float2* gathered, int world, int rows, int K, float2* cand, int* cnt,
                         cudaStream_t s);
// As launch_dh_reduce_bf16 with an fp32 result (the vocabulary-parallel all-reduce's
// buffer), launched the ordinary way. n_elem % 8 == 0.
void launch_dh_reduce_f32(const float* dHp, int n_split, int64_t n_elem, float* out, int d,
                          const float4* cst, cudaStream_t s);
void launch_f32_to_bf16(const float* in, int64_t n_elem, uint16_t* out, cudaStream_t s);
// Teacher top-K cache: per row, the threshold = the K-th best of the n_vt tile
// bests (logit descending, id ascending), or "take everything" when n_vt <= K.
void launch_topk_threshold(const float2* tbest, int n_vt, int rows, int K, float2* theta,
                           cudaStream_t s);
// Per row, the K best candidates in descending order -> idx, logit (row stride K).
void launch_topk_select(const float2* cand, const int* cnt, int cap, int rows, int K,
                        int32_t* idx_out, float* logit_out, unsigned* status, cudaStream_t s);
void launch_loss_finalize(const float* ell_all, const uint8_t* mask, int64_t T, Misc* misc,
                          float* loss, cudaStream_t s);

// ---- fp32 SIMT path (k_simt.cu)
void launch_simt_lse(const float* Hc, const float* W, int Tc, int V, int d, float2* part,
                     cudaStream_t s);
void launch_simt_grad(const float* Hc, const float* W, int Tc, int V, int d, const float4* cst,
                      float* G, int64_t ldG, cudaStream_t s);
// C[m][n] = (beta ? C[m][n] : 0) + sum_k A[m*sam + k*sak] * B[n*sbn + k*sbk]
void launch_simt_gemm(const float* A, int64_t sam, int64_t sak, const float* B, int64_t sbn,
                      int64_t sbk, float* C, int64_t ldc, int M, int N, int Kd, int beta,
                      cudaStream_t s);
constexpr int kSimtTile = 64;

// ---- bf16 tcgen05 path (k_tc.cu): declared in k_tc.h
}  // namespace ckl
