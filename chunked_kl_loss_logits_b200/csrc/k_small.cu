// Memory-bound kernels of the fused top-K forward-KL loss: the sparse teacher
// term (a warp per token: teacher softmax, merged probabilities, entropy, and
// the ids sorted for the forward contraction; the fp32 path also gathers the
// student logits at the K cached ids by dot products), the
// merge of per-vocabulary-tile log-sum-exp partials, the top-K correction of the
// gradient tile, the split-K reduction of dH, and the mask count / loss mean.
//
// The per-token loss follows "Chunked KL loss, running Knowledge Distillation
// locally in less <6GB VRAM" (README formula section):
//   l_t = sum_{v in S} P_v log P_v - sum_{v in S} P_v z_v + M logsumexp(z)
// where only the last term spans the vocabulary; the first two need the K
// cached entries only.
#include <math.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace ckl {

namespace {

constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Dot product of two 16-byte vectors of fp32 (the fp32 gather path).
__device__ __forceinline__ float dot16(const uint4& a, const uint4& b, const float*) {
  return __uint_as_float(a.x) * __uint_as_float(b.x) + __uint_as_float(a.y) * __uint_as_float(b.y) +
         __uint_as_float(a.z) * __uint_as_float(b.z) + __uint_as_float(a.w) * __uint_as_float(b.w);
}

constexpr int kGatherWarps = 4;
constexpr int kTeacherWarps = 8;
constexpr int kReduceBlock = 512;  // dH split reduction: threads per block

__host__ __device__ __forceinline__ int pow2_at_least(int k) {
  int p = 1;
  while (p < k) p <<= 1;
  return p;
}
// Shared memory of one teacher warp: ids and logits (k_bytes each), then the sort keys.
__host__ __device__ __forceinline__ size_t teacher_warp_bytes(int K, int k_bytes) {
  return 2 * (size_t)k_bytes + 8 * (size_t)pow2_at_least(K);
}

// One warp per token of the chunk (bf16 path):
//  1. stage the token's K ids and logits (16-byte loads when K % 4 == 0)
//  2. p = softmax(logits); M = sum p; P_k = total p of slot k's id (repeats add)
//  3. ent = sum_k p_k log P_k
//  4. the (id, p) pairs in ascending id order (ties in slot order), for the
//     forward contraction's epilogue to pick z at the ids and form sum_k p_k z_k
// Ids are checked against the full vocabulary V_all; the sorted ids are written
// relative to v0, the first row of this caller's slice of the LM head (0 unless
// the vocabulary is split over ranks), so ids outside the slice match no column.
__device__ __forceinline__ void teacher_token(
    unsigned char* smem, const int32_t* __restrict__ idx, const float* __restrict__ logit,
    int64_t t0, int Tc, int V_all, int v0, int V_loc, int K, int k_bytes,
    float4* __restrict__ tok, float* __restrict__ Pk_out, int32_t* __restrict__ sid_out,
    float* __restrict__ sp_out, unsigned* status, const uint16_t* __restrict__ Hc,
    const uint16_t* __restrict__ W, int d, int* __restrict__ rep) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kTeacherWarps + warp;
  if (rep && blockIdx.x == 0 && threadIdx.x == 0) rep[0] = 0;  // this chunk's repair list
  if (i >= Tc) return;
  const int64_t t = t0 + i;
  int* sId = reinterpret_cast<int*>(smem + (size_t)warp * teacher_warp_bytes(K, k_bytes));
  float* sP = reinterpret_cast<float*>(smem + (size_t)warp * teacher_warp_bytes(K, k_bytes) +
                                       k_bytes);

  const int32_t* idr = idx + t * K;
  const float* lgr = logit + t * K;
  if ((K & 3) == 0) {
    for (int k4 = lane; k4 < (K >> 2); k4 += 32) {
      reinterpret_cast<int4*>(sId)[k4] = __ldg(reinterpret_cast<const int4*>(idr) + k4);
      reinterpret_cast<float4*>(sP)[k4] = __ldg(reinterpret_cast<const float4*>(lgr) + k4);
    }
  } else {
    for (int k = lane; k < K; k += 32) {
      sId[k] = __ldg(idr + k);
      sP[k] = __ldg(lgr + k);
    }
  }
  __syncwarp();
  // Reference logit of the stored-exp backward: the student's logit (log2 units) at
  // the slot with the largest teacher logit among the ids of this caller's rows,
  // -inf when there is none. A logit at an actual id is at most the row's maximum,
  // so exp(z - reference) can only overflow when the maximum lies far above it,
  // which the forward epilogue checks tile by tile.
  float r2 = 0.f;
  if (Hc) {
    float best = -INFINITY;
    int bslot = K;
    for (int k = lane; k < K; k += 32) {
      const int id = sId[k] - v0;
      if (id >= 0 && id < V_loc && sP[k] > best) { best = sP[k]; bslot = k; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int os = __shfl_xor_sync(0xffffffffu, bslot, o);
      if (ob > best || (ob == best && os < bslot)) { best = ob; bslot = os; }
    }
    if (bslot < K) {
      // four 16-byte pieces of each row in flight per lane, four partial sums
      const uint4* hr = reinterpret_cast<const uint4*>(Hc + (int64_t)i * d);
      const uint4* wr = reinterpret_cast<const uint4*>(W + (int64_t)(sId[bslot] - v0) * d);
      const int n16 = d >> 3;
      float zq[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c0 = lane; c0 < n16; c0 += 128) {
        uint4 a[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + 32 * u;
          a[u] = c < n16 ? __ldg(hr + c) : make_uint4(0, 0, 0, 0);
          b[u] = c < n16 ? __ldg(wr + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float z = zq[u];
          z = fmaf(lo_bf16(a[u].x), lo_bf16(b[u].x), z); z = fmaf(hi_bf16(a[u].x), hi_bf16(b[u].x), z);
          z = fmaf(lo_bf16(a[u].y), lo_bf16(b[u].y), z); z = fmaf(hi_bf16(a[u].y), hi_bf16(b[u].y), z);
          z = fmaf(lo_bf16(a[u].z), lo_bf16(b[u].z), z); z = fmaf(hi_bf16(a[u].z), hi_bf16(b[u].z), z);
          z = fmaf(lo_bf16(a[u].w), lo_bf16(b[u].w), z); z = fmaf(hi_bf16(a[u].w), hi_bf16(b[u].w), z);
          zq[u] = z;
        }
      }
      r2 = warp_sum((zq[0] + zq[1]) + (zq[2] + zq[3])) * 1.4426950408889634f;
    } else {
      r2 = -INFINITY;
    }
  }
  float mx = -INFINITY;
  for (int k = lane; k < K; k += 32) mx = fmaxf(mx, sP[k]);
  mx = warp_max(mx);
  const bool live = mx > -INFINITY;
  float se = 0.f;
  for (int k = lane; k < K; k += 32) se += live ? expf(sP[k] - mx) : 0.f;
  se = warp_sum(se);
  __syncwarp();
  for (int k = lane; k < K; k += 32) {
    sP[k] = (live && se > 0.f) ? expf(sP[k] - mx) / se : 0.f;
    const int id = sId[k];
    if (id < 0 || id >= V_all) atomicOr(status, (unsigned)ST_INDEX_RANGE);
  }
  // Sort the (id, slot) pairs by id, ties in slot order: a bitonic network over the
  // next power of two >= K of 64-bit keys (signed id, sign bit flipped, above the
  // slot; padding keys sort last). The sorted order is what the forward epilogue
  // walks, and equal ids become runs whose first slot carries their pooled P.
  unsigned long long* key = reinterpret_cast<unsigned long long*>(
      smem + (size_t)warp * teacher_warp_bytes(K, k_bytes) + 2 * k_bytes);
  const int Pk2 = pow2_at_least(K);
  for (int k = lane; k < Pk2; k += 32)
    key[k] = k < K ? ((unsigned long long)((uint32_t)sId[k] ^ 0x80000000u) << 32) | (uint32_t)k
                   : ~0ull;
  __syncwarp();
  for (int size = 2; size <= Pk2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int j = lane; j < Pk2; j += 32) {
        const int partner = j ^ stride;
        if (partner > j) {
          const unsigned long long a = key[j], b = key[partner];
          if ((a > b) == ((j & size) == 0)) {
            key[j] = b;
            key[partner] = a;
          }
        }
      }
      __syncwarp();
    }
  }
  // Per sorted position: the run of equal ids around it (one entry unless an id
  // repeats), its pooled probability P (summed in slot order), the sorted outputs,
  // and P per slot for the entropy term (kept in sId's place, no longer needed).
  float* sMP = reinterpret_cast<float*>(sId);
  for (int j = lane; j < K; j += 32) {
    const uint32_t hi = (uint32_t)(key[j] >> 32);
    const int slot = (int)(uint32_t)key[j];
    int st = j;
    while (st > 0 && (uint32_t)(key[st - 1] >> 32) == hi) --st;
    float P = 0.f;
    for (int m = st; m < K && (uint32_t)(key[m] >> 32) == hi; ++m) P += sP[(uint32_t)key[m]];
    const float p = sP[slot];
    sMP[slot] = P;
    Pk_out[(int64_t)i * K + slot] = st == j ? P : 0.f;
    sid_out[(int64_t)i * K + j] = (int)(hi ^ 0x80000000u) - v0;
    sp_out[(int64_t)i * K + j] = p;
  }
  __syncwarp();
  float ent = 0.f, Msum = 0.f;
  for (int k = lane; k < K; k += 32) {
    const float p = sP[k];
    if (p > 0.f) ent += p * logf(sMP[k]);
    Msum += p;
  }
  ent = warp_sum(ent);
  Msum = warp_sum(Msum);
  if (lane == 0) tok[i] = make_float4(ent, 0.f, Msum, r2);
}

// The next chunk's teacher statistics may run behind the current chunk's dH
// contraction as a dependent launch (two blocks beside each of its CTAs); they
// touch none of that kernel's inputs or outputs. One thread then waits for the dH
// kernel to complete, so that this kernel's completion still orders the dW
// contraction and everything after it behind both.
__global__ void __launch_bounds__(kTeacherWarps * 32) teacher_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ logit, int64_t t0, int Tc,
    int V_all, int v0, int V_loc, int K, int k_bytes, float4* __restrict__ tok,
    float* __restrict__ Pk_out, int32_t* __restrict__ sid_out, float* __restrict__ sp_out,
    unsigned* status, const uint16_t* __restrict__ Hc, const uint16_t* __restrict__ W, int d,
    int* __restrict__ rep) {
  extern __shared__ __align__(16) unsigned char smem[];
  teacher_token(smem, idx, logit, t0, Tc, V_all, v0, V_loc, K, k_bytes, tok, Pk_out, sid_out,
                sp_out, status, Hc, W, d, rep);
  if (blockIdx.x == 0 && threadIdx.x == 0) griddep_wait();
}

// One warp per token of the chunk.
//  1. stage the token's K ids and logits (16-byte loads when K % 4 == 0) and H row
//  2. p = softmax(logits); M = sum p; P_k = total p of slot k's id (repeats add)
//  3. ent = sum_k p_k log P_k
//  4. z_k = H_t . W[id_k] for every slot, 4 rows in flight per lane
//  5. cross = sum_k p_k z_k
template <typename Tin>
__global__ void __launch_bounds__(kGatherWarps * 32) gather_kernel(
    const Tin* __restrict__ H, const Tin* __restrict__ W, const int32_t* __restrict__ idx,
    const float* __restrict__ logit, int64_t t0, int Tc, int d, int V, int K, int h_bytes,
    int k_bytes, float4* __restrict__ tok, float* __restrict__ zk_out, float* __restrict__ Pk_out,
    unsigned* status) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kGatherWarps + warp;
  if (i >= Tc) return;
  const int64_t t = t0 + i;
  unsigned char* base = smem + (size_t)warp * (h_bytes + 2 * k_bytes);
  uint4* sH = reinterpret_cast<uint4*>(base);
  int* sId = reinterpret_cast<int*>(base + h_bytes);
  float* sP = reinterpret_cast<float*>(base + h_bytes + k_bytes);

  // 1. stage ids, logits (into sP for now) and the H row
  const int32_t* idr = idx + t * K;
  const float* lgr = logit + t * K;
  if ((K & 3) == 0) {
    for (int k4 = lane; k4 < (K >> 2); k4 += 32) {
      reinterpret_cast<int4*>(sId)[k4] = __ldg(reinterpret_cast<const int4*>(idr) + k4);
      reinterpret_cast<float4*>(sP)[k4] = __ldg(reinterpret_cast<const float4*>(lgr) + k4);
    }
  } else {
    for (int k = lane; k < K; k += 32) {
      sId[k] = __ldg(idr + k);
      sP[k] = __ldg(lgr + k);
    }
  }
  constexpr int VEC = 16 / sizeof(Tin);
  const int nvec = d / VEC;
  const uint4* Hr = reinterpret_cast<const uint4*>(H + t * d);
  for (int v = lane; v < nvec; v += 32) sH[v] = __ldg(Hr + v);
  __syncwarp();

  // 2. teacher softmax over the cached logits
  float mx = -INFINITY;
  for (int k = lane; k < K; k += 32) mx = fmaxf(mx, sP[k]);
  mx = warp_max(mx);
  const bool live = mx > -INFINITY;
  float se = 0.f;
  for (int k = lane; k < K; k += 32) se += live ? expf(sP[k] - mx) : 0.f;
  se = warp_sum(se);
  __syncwarp();
  for (int k = lane; k < K; k += 32) {
    const float p = (live && se > 0.f) ? expf(sP[k] - mx) / se : 0.f;
    sP[k] = p;
    const int id = sId[k];
    if (id < 0 || id >= V) atomicOr(status, (unsigned)ST_INDEX_RANGE);
  }
  __syncwarp();

  // 3. merged probabilities and the teacher entropy term
  float ent = 0.f, Msum = 0.f;
  for (int k = lane; k < K; k += 32) {
    const int id = sId[k];
    const float p = sP[k];
    float P = 0.f;
    bool first = true;
    for (int j = 0; j < K; ++j) {
      if (sId[j] == id) {
        P += sP[j];
        first = first && (j >= k);
      }
    }
    if (p > 0.f) ent += p * logf(P);
    Msum += p;
    Pk_out[(int64_t)i * K + k] = first ? P : 0.f;
  }
  ent = warp_sum(ent);
  Msum = warp_sum(Msum);

  // 4-5. student logits at the cached ids and the cross term
  float cross = 0.f;
  const Tin* tag = nullptr;
  constexpr int R = 8;  // W rows in flight per warp
  for (int k0 = 0; k0 < K; k0 += R) {
    const uint4* row[R];
    bool ok[R];
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int k = k0 + u;
      const int id = k < K ? sId[k] : -1;
      ok[u] = k < K && id >= 0 && id < V;
      row[u] = reinterpret_cast<const uint4*>(W + (int64_t)(ok[u] ? id : 0) * d);
    }
    float acc[R];
#pragma unroll
    for (int u = 0; u < R; ++u) acc[u] = 0.f;
    int v = lane;
    for (; v + 32 < nvec; v += 64) {
      const uint4 h0 = sH[v], h1 = sH[v + 32];
      uint4 w0[R], w1[R];
#pragma unroll
      for (int u = 0; u < R; ++u) {
        if (ok[u]) {
          w0[u] = __ldg(row[u] + v);
          w1[u] = __ldg(row[u] + v + 32);
        }
      }
#pragma unroll
      for (int u = 0; u < R; ++u)
        if (ok[u]) acc[u] += dot16(h0, w0[u], tag) + dot16(h1, w1[u], tag);
    }
    if (v < nvec) {
      const uint4 h0 = sH[v];
#pragma unroll
      for (int u = 0; u < R; ++u)
        if (ok[u]) acc[u] += dot16(h0, __ldg(row[u] + v), tag);
    }
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const float z = warp_sum(acc[u]);
      const int k = k0 + u;
      if (k < K) {
        const float p = sP[k];
        if (p > 0.f) cross += p * z;
        if (lane == 0) zk_out[(int64_t)i * K + k] = z;
      }
    }
  }
  if (lane == 0) tok[i] = make_float4(ent, cross, Msum, 0.f);
}

constexpr int kCombTok = 16, kCombSplit = 64;

// From a token's merged (max, sum) in log2 units and its cross term: lse,
// l_t = ent - cross + M lse and the gradient multipliers.
// With `rep` (stored-exp backward): the row's reference R for the stored exp(z - R),
// in log2 units, is the teacher kernel's reference r2 unless some tile of this
// caller's rows has its maximum more than kRefGap above r2 (local_M2, the largest
// tile maximum, tells); such a tile stored exp(z - its own maximum), so the row
// joins the repair list and R becomes local_M2. cst.w = R.
__device__ __forceinline__ void finish_token(int64_t t0, int i, float M2, float S, float cross,
                                             const uint8_t* __restrict__ mask,
                                             const float4* __restrict__ tok,
                                             const Misc* __restrict__ misc, float4* __restrict__ cst,
                                             float* __restrict__ lse_all,
                                             float* __restrict__ ell_all, float local_M2,
                                             int* __restrict__ rep) {
  const float lse = (M2 + log2f(S)) * kLn2;
  const float4 t4 = tok[i];
  const float ell = t4.x - cross + t4.z * lse;
  const int64_t t = t0 + i;
  const float sc = (mask == nullptr || mask[t] != 0) ? misc->invN : 0.f;
  float R = 0.f;
  if (rep) {
    R = t4.w;
    if (local_M2 > t4.w + kRefGap) {
      R = local_M2;
      rep[1 + atomicAdd(rep, 1)] = i;
    }
  }
  cst[i] = make_float4(lse, sc * t4.z, sc, R);
  lse_all[t] = lse;
  ell_all[t] = ell;
}

// Merge the per-vocabulary-tile (max, sum) partials into logsumexp(z_t), then
// l_t = ent - cross + M lse and the gradient multipliers. A block covers 16
// tokens; its 64 thread groups of 16 each merge every 64th vocabulary tile
// (coalesced 128-byte reads of 16 consecutive tokens), then 16 threads merge the 64
// results (128 blocks per 2048-token chunk, so every SM takes part).
// With `stats` set (vocabulary split over ranks) it stops at this rank's
// (max, sum, cross) per token; vp_merge_kernel finishes after the exchange.
__global__ void __launch_bounds__(kCombTok * kCombSplit) combine_kernel(
    int64_t t0, int Tc, int n_vt, const uint8_t* __restrict__ mask,
    const float2* __restrict__ part, const float* __restrict__ xpart,
    const float4* __restrict__ tok, const Misc* __restrict__ misc,
    float4* __restrict__ cst, float* __restrict__ lse_all, float* __restrict__ ell_all,
    float4* __restrict__ stats, int* __restrict__ rep) {
  __shared__ float sm[kCombSplit][kCombTok], ss[kCombSplit][kCombTok], sx[kCombSplit][kCombTok];
  const int tk = threadIdx.x % kCombTok, sp = threadIdx.x / kCombTok;
  const int i = blockIdx.x * kCombTok + tk;
  float m2 = -INFINITY, s = 0.f, x = 0.f;
  if (i < Tc) {
#pragma unroll 4
    for (int j = sp; j < n_vt; j += kCombSplit) {
      const float2 q = part[(int64_t)j * Tc + i];
      if (q.x > m2) {
        s = s * ex2_approx(m2 - q.x) + q.y;
        m2 = q.x;
      } else {
        s += q.y * ex2_approx(q.x - m2);
      }
      if (xpart) x += xpart[(int64_t)j * Tc + i];
    }
  }
  sm[sp][tk] = m2;
  ss[sp][tk] = s;
  sx[sp][tk] = x;
  __syncthreads();
  if (sp != 0 || i >= Tc) return;
  float M2 = -INFINITY;
#pragma unroll
  for (int j = 0; j < kCombSplit; ++j) M2 = fmaxf(M2, sm[j][tk]);
  float S = 0.f, X = 0.f;
#pragma unroll
  for (int j = 0; j < kCombSplit; ++j) {
    if (sm[j][tk] > -INFINITY) S += ss[j][tk] * ex2_approx(sm[j][tk] - M2);
    X += sx[j][tk];
  }
  const float cross = xpart ? X : tok[i].y;  // bf16: from the contraction's epilogue; fp32: gathered
  if (stats) {
    stats[i] = make_float4(M2, S, cross, 0.f);
    return;
  }
  finish_token(t0, i, M2, S, cross, mask, tok, misc, cst, lse_all, ell_all, M2, rep);
}

// Vocabulary split over ranks: merge every rank's (max, sum, cross) of a token,
// in rank order (stats_all is rank-major, world x Tc), so that every rank
// computes the same lse and l_t bit for bit. One thread per token.
__global__ void vp_merge_kernel(int64_t t0, int Tc, int world, int rank,
                                const float4* __restrict__ stats_all,
                                const uint8_t* __restrict__ mask, const float4* __restrict__ tok,
                                const Misc* __restrict__ misc, float4* __restrict__ cst,
                                float* __restrict__ lse_all, float* __restrict__ ell_all,
                                int* __restrict__ rep) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= Tc) return;
  float M2 = -INFINITY;
  for (int r = 0; r < world; ++r) M2 = fmaxf(M2, stats_all[(int64_t)r * Tc + i].x);
  float S = 0.f, X = 0.f;
  for (int r = 0; r < world; ++r) {
    const float4 q = stats_all[(int64_t)r * Tc + i];
    if (q.x > -INFINITY) S += q.y * ex2_approx(q.x - M2);
    X += q.z;
  }
  // the reference and the stored exps are this rank's own: its rows' largest tile max
  finish_token(t0, i, M2, S, X, mask, tok, misc, cst, lse_all, ell_all,
               stats_all[(int64_t)rank * Tc + i].x, rep);
}

// Stored-exp backward, rows on the repair list: the forward epilogue stored
// exp2(z log2e - ref_j) in each vocabulary tile j, with ref_j the tile's maximum m2_j
// when m2_j > r2 + kRefGap and the row's reference r2 otherwise; the row's common
// reference is now R = cst.w (the largest tile maximum), so every stored value is
// multiplied by exp2(ref_j - R) <= 1, in place. Rows not on the list need nothing.
// A fixed grid strides over (listed rows) x (64-wide vocabulary blocks) x 8 groups
// of 8 elements; with an empty list every thread reads the count and returns.
__global__ void __launch_bounds__(256) repair_kernel(uint16_t* __restrict__ G, int n_vb, int Tc,
                                                     int V, const float2* __restrict__ part,
                                                     const float4* __restrict__ cst,
                                                     const float4* __restrict__ tok,
                                                     const int* __restrict__ rep) {
  const int n = rep[0];
  const int64_t per_row = (int64_t)n_vb * 8;
  const int64_t total = (int64_t)n * per_row;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < total;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(it / per_row);
    const int rem = (int)(it - (int64_t)r * per_row);
    const int vb = rem >> 3, c = (rem & 7) * 8;
    const int v = vb * 64 + c;
    if (v >= V) continue;
    const int t = rep[1 + r];
    const float R = cst[t].w, r2 = tok[t].w;
    const float m2 = part[(int64_t)(v >> 8) * Tc + t].x;
    const float f = ex2_approx((m2 > r2 + kRefGap ? m2 : r2) - R);
    uint4* q = reinterpret_cast<uint4*>(G + (((int64_t)(t >> 6) * n_vb + vb) << 12) +
                                        ((t & 63) << 6) + c);
    uint4 y = *q;
    y.x = pack_bf16x2(lo_bf16(y.x) * f, hi_bf16(y.x) * f);
    y.y = pack_bf16x2(lo_bf16(y.y) * f, hi_bf16(y.y) * f);
    y.z = pack_bf16x2(lo_bf16(y.z) * f, hi_bf16(y.z) * f);
    y.w = pack_bf16x2(lo_bf16(y.w) * f, hi_bf16(y.w) * f);
    *q = y;
  }
}

// Element (i, id) of the gradient buffer: fp32 row-major (ldG), bf16 blocked
// (64 x 64 blocks, ld = the number of 64-wide vocabulary blocks).
__device__ __forceinline__ int64_t g_off(const float*, int64_t i, int id, int64_t ld) {
  return i * ld + id;
}
__device__ __forceinline__ int64_t g_off(const uint16_t*, int64_t i, int id, int64_t ld) {
  return (((i >> 6) * ld + (id >> 6)) << 12) + ((i & 63) << 6) + (id & 63);
}
__device__ __forceinline__ void store_g(float* G, int64_t off, float v) { G[off] = v; }
__device__ __forceinline__ void store_g(uint16_t* G, int64_t off, float v) {
  G[off] = f32_to_bf16(v);
}
__device__ __forceinline__ float load_g(const float* G, int64_t off) { return G[off]; }
__device__ __forceinline__ float load_g(const uint16_t* G, int64_t off) {
  return bf16_to_f32(G[off]);
}

// One thread per (token, slot) that holds the first occurrence of an id (P_k > 0).
// G holds gmul exp(z - lse): G[i][id] -= s P_k. With `row_ref` G holds the stored
// exp(z - R) instead, the gradient being c exp(z - R) with c = gmul exp(R - lse):
// G[i][id] -= (P_k / M) exp(lse - R), so that c times it is the gradient there.
// Ids are taken relative to v0 (the slice's first row); ids outside [0, V) of
// the slice belong to another rank and are skipped.
template <typename Tg>
__global__ void fixup_kernel(const int32_t* __restrict__ idx, int64_t t0, int Tc, int K, int V,
                             int v0, int64_t ldG, const float4* __restrict__ cst,
                             const float4* __restrict__ tok, const float* __restrict__ Pk, Tg* G,
                             int row_ref) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)Tc * K) return;
  const float P = Pk[e];
  if (!(P > 0.f)) return;
  const int64_t i = e / K;
  const int id = idx[t0 * K + e] - v0;
  if (id < 0 || id >= V) return;
  const float4 c = cst[i];
  const int64_t off = g_off(G, i, id, ldG);
  const float sub = row_ref ? (P / tok[i].z) * ex2_approx(c.x * 1.4426950408889634f - c.w)
                            : c.z * P;
  store_g(G, off, load_g(G, off) - sub);
}

// Sum of the split-K partials in fp32 (vocabulary split over ranks: the ranks'
// sums are added by the exchange before the conversion to bf16); each row times
// its row factor (1 without cst).
__global__ void dh_reduce_f32_kernel(const float* __restrict__ dHp, int n_split, int64_t n_elem,
                                     float* __restrict__ out, int d, const float4* __restrict__ cst) {
  const int64_t e8 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (e8 >= n_elem) return;
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < n_split; ++s) {
    const float4* p = reinterpret_cast<const float4*>(dHp + s * n_elem + e8);
    const float4 x = p[0], y = p[1];
    a[0] += x.x; a[1] += x.y; a[2] += x.z; a[3] += x.w;
    a[4] += y.x; a[5] += y.y; a[6] += y.z; a[7] += y.w;
  }
  const float c = row_factor(cst, e8 / d);
  float4* o = reinterpret_cast<float4*>(out + e8);
  o[0] = make_float4(a[0] * c, a[1] * c, a[2] * c, a[3] * c);
  o[1] = make_float4(a[4] * c, a[5] * c, a[6] * c, a[7] * c);
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ in, int64_t n_elem,
                                   uint16_t* __restrict__ out) {
  const int64_t e4 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (e4 >= n_elem) return;
  const float4 x = *reinterpret_cast<const float4*>(in + e4);
  uint2 o;
  o.x = pack_bf16x2(x.x, x.y);
  o.y = pack_bf16x2(x.z, x.w);
  *reinterpret_cast<uint2*>(out + e4) = o;
}

// Sum of the split-K partials -> bf16 dH, each row times its row factor, over a
// grid that strides the chunk (one block per SM). It may run behind the dW
// contraction as a dependent launch (one block beside each of that kernel's CTAs):
// one thread then waits for the dW kernel to complete, so this kernel's completion
// still orders everything after it behind both.
__global__ void __launch_bounds__(kReduceBlock) dh_reduce_bf16_kernel(
    const float* __restrict__ dHp, int n_split, int64_t n_elem, uint16_t* __restrict__ dH, int d,
    const float4* __restrict__ cst) {
  // Per thread and round: U groups of 8 elements; the partials of up to SG splits are
  // loaded together before they are added (in split order). U = 1 keeps a block within
  // the registers the dW contraction's CTA leaves on its SM.
  constexpr int U = 1, SG = 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x * 8;
  for (int64_t e0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; e0 < n_elem;
       e0 += U * stride) {
    float a[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int k = 0; k < 8; ++k) a[u][k] = 0.f;
    for (int s0 = 0; s0 < n_split; s0 += SG) {
      float4 x[SG][U], y[SG][U];
#pragma unroll
      for (int g = 0; g < SG; ++g)
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int64_t e8 = e0 + u * stride;
          x[g][u] = y[g][u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (s0 + g < n_split && e8 < n_elem) {
            const float4* p = reinterpret_cast<const float4*>(dHp + (s0 + g) * n_elem + e8);
            x[g][u] = p[0];
            y[g][u] = p[1];
          }
        }
#pragma unroll
      for (int g = 0; g < SG; ++g)
#pragma unroll
        for (int u = 0; u < U; ++u) {
          if (s0 + g < n_split) {
            a[u][0] += x[g][u].x; a[u][1] += x[g][u].y; a[u][2] += x[g][u].z; a[u][3] += x[g][u].w;
            a[u][4] += y[g][u].x; a[u][5] += y[g][u].y; a[u][6] += y[g][u].z; a[u][7] += y[g][u].w;
          }
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t e8 = e0 + u * stride;
      if (e8 >= n_elem) continue;
      if (cst) {
        const float c = row_factor(cst, e8 / d);
#pragma unroll
        for (int k = 0; k < 8; ++k) a[u][k] *= c;
      }
      uint4 o;
      o.x = pack_bf16x2(a[u][0], a[u][1]);
      o.y = pack_bf16x2(a[u][2], a[u][3]);
      o.z = pack_bf16x2(a[u][4], a[u][5]);
      o.w = pack_bf16x2(a[u][6], a[u][7]);
      *reinterpret_cast<uint4*>(dH + e8) = o;
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) griddep_wait();
}

// ------------------------------------------------------------ teacher top-K cache
// Candidates are ordered by (logit descending, id ascending), encoded in one
// 64-bit key: the float's order-preserving bits above the complemented id.
__device__ __forceinline__ unsigned long long topk_key(float v, int id) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)id);
}
__device__ __forceinline__ float topk_key_value(unsigned long long k) {
  const uint32_t u = (uint32_t)(k >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}
__device__ __forceinline__ int topk_key_id(unsigned long long k) {
  return (int)(0xFFFFFFFFu - (uint32_t)k);
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kThreshWarps = 8;
constexpr int kThreshRegKeys = 32;  // keys per lane kept in registers (n_vt <= 1024)

// Warp per row: the K-th best of the row's n_vt tile bests, by binary search on
// the key bits (the largest key x with at least K keys >= x). Every one of the
// row's K best logits is at least as good as it, and only the K tiles whose best
// beats it can hold such logits, so at most K * 256 candidates follow.
__global__ void __launch_bounds__(kThreshWarps * 32) topk_threshold_kernel(
    const float2* __restrict__ tbest, int n_vt, int rows, int K, float2* __restrict__ theta) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kThreshWarps + warp;
  if (i >= rows) return;
  if (n_vt <= K) {  // every tile may hold top-K entries: take everything
    if (lane == 0) theta[i] = make_float2(-INFINITY, __int_as_float(INT_MAX));
    return;
  }
  const bool in_regs = n_vt <= 32 * kThreshRegKeys;
  unsigned long long keys[kThreshRegKeys];
#pragma unroll
  for (int r = 0; r < kThreshRegKeys; ++r) {
    const int j = r * 32 + lane;
    keys[r] = 0;
    if (in_regs && j < n_vt) {
      const float2 b = tbest[(int64_t)j * rows + i];
      keys[r] = topk_key(b.x, __float_as_int(b.y));
    }
  }
  unsigned long long prefix = 0;
  for (int bit = 63; bit >= 0; --bit) {
    const unsigned long long cand = prefix | (1ull << bit);
    int c = 0;
    if (in_regs) {
#pragma unroll
      for (int r = 0; r < kThreshRegKeys; ++r) c += keys[r] >= cand;
    } else {
      for (int j = lane; j < n_vt; j += 32) {
        const float2 b = tbest[(int64_t)j * rows + i];
        c += topk_key(b.x, __float_as_int(b.y)) >= cand;
      }
    }
    if (warp_sum_int(c) >= K) prefix = cand;
  }
  if (lane == 0) theta[i] = make_float2(topk_key_value(prefix), __int_as_float(topk_key_id(prefix)));
}

constexpr int kSelectThreads = 256;

// Block per row: the K best of the row's candidates (by the same bit search over
// the count of keys at least as good), then a bitonic sort into descending order.
__global__ void __launch_bounds__(kSelectThreads) topk_select_kernel(
    const float2* __restrict__ cand, const int* __restrict__ cnt, int cap, int rows, int K,
    int32_t* __restrict__ idx_out, float* __restrict__ logit_out, unsigned* status) {
  __shared__ unsigned long long sel[1024];
  __shared__ int wsum[kSelectThreads / 32];
  __shared__ int nsel;
  const int i = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int c = cnt[i];
  if (c > cap) {  // cannot happen (at most K * 256 candidates); keep the first cap
    if (tid == 0) atomicOr(status, (unsigned)ST_INTERNAL);
    c = cap;
  }
  const float2* crow = cand + (int64_t)i * cap;
  unsigned long long prefix = 0;
  for (int bit = 63; bit >= 0; --bit) {
    const unsigned long long want = prefix | (1ull << bit);
    int n = 0;
    for (int j = tid; j < c; j += kSelectThreads) {
      const float2 e = crow[j];
      n += topk_key(e.x, __float_as_int(e.y)) >= want;
    }
    n = warp_sum_int(n);
    if (lane == 0) wsum[warp] = n;
    __syncthreads();
    int total = 0;
#pragma unroll
    for (int w = 0; w < kSelectThreads / 32; ++w) total += wsum[w];
    __syncthreads();
    if (total >= K) prefix = want;
  }
  int P = 1;
  while (P < K) P <<= 1;
  if (tid == 0) nsel = 0;
  for (int j = tid; j < P; j += kSelectThreads) sel[j] = 0;  // padding sorts last
  __syncthreads();
  for (int j = tid; j < c; j += kSelectThreads) {
    const float2 e = crow[j];
    const unsigned long long k = topk_key(e.x, __float_as_int(e.y));
    if (k >= prefix) {
      const int slot = atomicAdd(&nsel, 1);
      if (slot < K) sel[slot] = k;
    }
  }
  __syncthreads();
  // bitonic sort of sel[0, P) into descending key order
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int j = tid; j < P; j += kSelectThreads) {
        const int partner = j ^ stride;
        if (partner > j) {
          const bool desc = (j & size) == 0;
          const unsigned long long a = sel[j], b = sel[partner];
          if (desc ? (a < b) : (a > b)) {
            sel[j] = b;
            sel[partner] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int k = tid; k < K; k += kSelectThreads) {
    idx_out[(int64_t)i * K + k] = topk_key_id(sel[k]);
    logit_out[(int64_t)i * K + k] = topk_key_value(sel[k]);
  }
}

constexpr int kReduceThreads = 1024;

__device__ double block_sum_d(double v, double* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  v = (threadIdx.x < (blockDim.x >> 5)) ? sh[threadIdx.x] : 0.0;
  if (warp == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  }
  return v;  // valid in thread 0
}

// Single block: N = number of tokens with mask != 0 (all tokens when mask is NULL).
__global__ void __launch_bounds__(kReduceThreads) mask_count_kernel(const uint8_t* mask, int64_t T,
                                                                     Misc* misc) {
  __shared__ double sh[32];
  double c = 0.0;
  if (mask == nullptr) {
    c = threadIdx.x == 0 ? (double)T : 0.0;
  } else {
    long long n = 0;
    for (int64_t t = threadIdx.x; t < T; t += blockDim.x) n += mask[t] != 0;
    c = (double)n;
  }
  c = block_sum_d(c, sh);
  if (threadIdx.x == 0) {
    misc->N = c;
    misc->loss_sum = 0.0;
    misc->invN = c > 0.0 ? (float)(1.0 / c) : 0.f;
  }
}

// Single block, fixed order: loss = sum_t mask_t l_t / N (0 when N == 0).
__global__ void __launch_bounds__(kReduceThreads) loss_finalize_kernel(
    const float* __restrict__ ell, const uint8_t* mask, int64_t T, Misc* misc, float* loss) {
  __shared__ double sh[32];
  double s = 0.0;
  for (int64_t t = threadIdx.x; t < T; t += blockDim.x)
    if (mask == nullptr || mask[t] != 0) s += (double)ell[t];
  s = block_sum_d(s, sh);
  if (threadIdx.x == 0) {
    misc->loss_sum = s;
    *loss = misc->N > 0.0 ? (float)(s / misc->N) : 0.f;
  }
}

inline unsigned blocks_for(int64_t n, int per) { return (unsigned)((n + per - 1) / per); }

// A kernel that runs beside the tensor-core kernels (as a dependent launch) asks for
// their shared-memory split, so an SM need not change it to take the kernel's
// blocks. Set once per device (`done`: one bit per device ordinal).
template <typename Kernel>
void prefer_max_shared(Kernel fn, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) == cudaSuccess)
    done.fetch_or(bit, std::memory_order_release);
}

}  // namespace

void launch_mask_count(const uint8_t* mask, int64_t T, Misc* misc, cudaStream_t s) {
  mask_count_kernel<<<1, kReduceThreads, 0, s>>>(mask, T, misc);
}

void launch_teacher(const int32_t* idx, const float* logit, int64_t t0, int Tc, int V_all, int v0,
                    int V_loc, int K, const ChunkBufs& b, unsigned* status, const uint16_t* Hc,
                    const uint16_t* W, int d, bool behind, cudaStream_t s) {
  const int k_bytes = (K * 4 + 15) & ~15;
  const size_t smem = (size_t)kTeacherWarps * teacher_warp_bytes(K, k_bytes);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(teacher_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  static std::atomic<uint64_t> carveout_set{0};
  prefer_max_shared(teacher_kernel, carveout_set);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks_for(Tc, kTeacherWarps));
  cfg.blockDim = dim3(kTeacherWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = behind ? 1 : 0;
  cudaLaunchKernelEx(&cfg, teacher_kernel, idx, logit, t0, Tc, V_all, v0, V_loc, K, k_bytes, b.tok,
                     b.Pk, b.sid, b.sp, status, Hc, W, d, Hc ? b.rep : nullptr);
}

template <typename Tin>
void launch_gather(const Tin* H, const Tin* W, const int32_t* idx, const float* logit, int64_t t0,
                   int Tc, int d, int V, int K, const ChunkBufs& b, unsigned* status,
                   cudaStream_t s) {
  const int h_bytes = (d * (int)sizeof(Tin) + 15) & ~15;
  const int k_bytes = (K * 4 + 15) & ~15;
  const size_t smem = (size_t)kGatherWarps * (h_bytes + 2 * k_bytes);
  // The attribute is per device: set it whenever the launch needs more than the default.
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(gather_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
  gather_kernel<Tin><<<blocks_for(Tc, kGatherWarps), kGatherWarps * 32, smem, s>>>(
      H, W, idx, logit, t0, Tc, d, V, K, h_bytes, k_bytes, b.tok, b.zk, b.Pk, status);
}
template void launch_gather<float>(const float*, const float*, const int32_t*, const float*,
                                   int64_t, int, int, int, int, const ChunkBufs&, unsigned*,
                                   cudaStream_t);

void launch_combine(int64_t t0, int Tc, int n_vt, const uint8_t* mask, const ChunkBufs& b,
                    float* lse_all, float* ell_all, float4* stats, bool row_ref, cudaStream_t s) {
  combine_kernel<<<blocks_for(Tc, kCombTok), kCombTok * kCombSplit, 0, s>>>(
      t0, Tc, n_vt, mask, b.part, b.xpart, b.tok, b.misc, b.cst, lse_all, ell_all, stats,
      row_ref ? b.rep : nullptr);
}

void launch_vp_merge(int64_t t0, int Tc, int world, int rank, const float4* stats_all,
                     const uint8_t* mask, const ChunkBufs& b, float* lse_all, float* ell_all,
                     bool row_ref, cudaStream_t s) {
  vp_merge_kernel<<<blocks_for(Tc, 128), 128, 0, s>>>(t0, Tc, world, rank, stats_all, mask, b.tok,
                                                      b.misc, b.cst, lse_all, ell_all,
                                                      row_ref ? b.rep : nullptr);
}

void launch_repair(uint16_t* G, int Tc, int V, const ChunkBufs& b, int num_sms, cudaStream_t s) {
  const int n_vb = (V + 63) / 64;
  repair_kernel<<<num_sms, 256, 0, s>>>(G, n_vb, Tc, V, b.part, b.cst, b.tok, b.rep);
}

template <typename Tg>
void launch_fixup(const int32_t* idx, int64_t t0, int Tc, int K, int V, int v0, int64_t ldG,
                  const ChunkBufs& b, bool row_ref, cudaStream_t s) {
  fixup_kernel<Tg><<<blocks_for((int64_t)Tc * K, 256), 256, 0, s>>>(
      idx, t0, Tc, K, V, v0, ldG, b.cst, b.tok, b.Pk, static_cast<Tg*>(b.G), row_ref ? 1 : 0);
}
template void launch_fixup<float>(const int32_t*, int64_t, int, int, int, int, int64_t,
                                  const ChunkBufs&, bool, cudaStream_t);
template void launch_fixup<uint16_t>(const int32_t*, int64_t, int, int, int, int, int64_t,
                                     const ChunkBufs&, bool, cudaStream_t);

void launch_dh_reduce_bf16(const float* dHp, int n_split, int64_t n_elem, uint16_t* dH, int d,
                           const float4* cst, int num_sms, cudaStream_t s) {
  const int64_t need = (n_elem / 8 + kReduceBlock - 1) / kReduceBlock;
  static std::atomic<uint64_t> carveout_set{0};
  prefer_max_shared(dh_reduce_bf16_kernel, carveout_set);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(need, num_sms)));
  cfg.blockDim = dim3(kReduceBlock);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, dh_reduce_bf16_kernel, dHp, n_split, n_elem, dH, d, cst);
}

void launch_dh_reduce_f32(const float* dHp, int n_split, int64_t n_elem, float* out, int d,
                          const float4* cst, cudaStream_t s) {
  dh_reduce_f32_kernel<<<blocks_for(n_elem / 8, 256), 256, 0, s>>>(dHp, n_split, n_elem, out, d,
                                                                   cst);
}

void launch_f32_to_bf16(const float* in, int64_t n_elem, uint16_t* out, cudaStream_t s) {
  f32_to_bf16_kernel<<<blocks_for(n_elem / 4, 256), 256, 0, s>>>(in, n_elem, out);
}

// Vocabulary split over ranks (top-K cache): this rank's K best of each row as
// (logit, global id) pairs, ids shifted by the rank's first row v0.
__global__ void topk_pack_kernel(const int32_t* __restrict__ idx, const float* __restrict__ lg,
                                 int64_t n, int v0, float2* __restrict__ out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e < n) out[e] = make_float2(lg[e], __int_as_float(idx[e] + v0));
}

// The gathered pairs are rank-major (world x rows x K); the select wants each
// row's world * K candidates together, with their count.
__global__ void topk_regroup_kernel(const float2* __restrict__ gathered, int world, int rows, int K,
                                    float2* __restrict__ cand, int* __restrict__ cnt) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t per_rank = (int64_t)rows * K;
  if (e >= per_rank * world) return;
  const int r = (int)(e / per_rank);
  const int64_t q = e - r * per_rank;
  const int row = (int)(q / K), k = (int)(q - (int64_t)row * K);
  cand[(int64_t)row * world * K + (int64_t)r * K + k] = gathered[e];
  if (r == 0 && k == 0) cnt[row] = world * K;
}

void launch_topk_pack(const int32_t* idx, const float* lg, int64_t n, int v0, float2* out,
                      cudaStream_t s) {
  topk_pack_kernel<<<blocks_for(n, 256), 256, 0, s>>>(idx, lg, n, v0, out);
}

void launch_topk_regroup(const float2* gathered, int world, int rows, int K, float2* cand, int* cnt,
                         cudaStream_t s) {
  topk_regroup_kernel<<<blocks_for((int64_t)world * rows * K, 256), 256, 0, s>>>(
      gathered, world, rows, K, cand, cnt);
}

void launch_topk_threshold(const float2* tbest, int n_vt, int rows, int K, float2* theta,
                           cudaStream_t s) {
  topk_threshold_kernel<<<blocks_for(rows, kThreshWarps), kThreshWarps * 32, 0, s>>>(
      tbest, n_vt, rows, K, theta);
}

void launch_topk_select(const float2* cand, const int* cnt, int cap, int rows, int K,
                        int32_t* idx_out, float* logit_out, unsigned* status, cudaStream_t s) {
  topk_select_kernel<<<rows, kSelectThreads, 0, s>>>(cand, cnt, cap, rows, K, idx_out, logit_out,
                                                     status);
}

// Self-test of the bounded pipeline wait: one thread waits, with the same bounded
// wait every pipeline kernel uses, on a freshly initialised mbarrier that nothing
// arrives at (its phase 0 never completes). The wait must give up after its bound,
// set ST_TIMEOUT and return; the kernel then exits. Completing is reported as
// ST_INTERNAL (it cannot happen).
__global__ void wait_bound_selftest_kernel(unsigned* status, long long* cycles) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  abort_flag = 0;
  const long long t0 = clock64();
  const bool completed = mbar_wait(&bar, 0u, &abort_flag, status);
  *cycles = clock64() - t0;
  if (completed) atomicOr(status, (unsigned)ST_INTERNAL);
}

void launch_wait_selftest(unsigned* status, long long* cycles, cudaStream_t s) {
  wait_bound_selftest_kernel<<<1, 32, 0, s>>>(status, cycles);
}

void launch_loss_finalize(const float* ell_all, const uint8_t* mask, int64_t T, Misc* misc,
                          float* loss, cudaStream_t s) {
  loss_finalize_kernel<<<1, kReduceThreads, 0, s>>>(ell_all, mask, T, misc, loss);
}

}  // namespace ckl
