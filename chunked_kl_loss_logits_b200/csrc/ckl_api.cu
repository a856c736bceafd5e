// C ABI of the fused, chunked top-K forward-KL loss: argument checks, the
// workspace plan, TMA descriptors, and the per-chunk launch sequence.
//
// Launch sequence of one ckl_fwd_bwd call (T tokens, `chunk` at a time), after
// the fused variant of "Chunked KL loss, running Knowledge Distillation locally
// in less <6GB VRAM" (README, "Full Chunked KL"):
//   mask_count                      N = sum(mask), 1/N
//   per chunk c (Tc tokens):
//     teacher                       p, merged P, sum P log P; ids sorted with their p (bf16)
//                                   (fp32: also z at the K ids and sum p z by dot products)
//     LSE contraction               per-vocabulary-tile (max, sum exp) of z = H_c W^T and
//                                   sum p z over the ids in the tile (bf16); stored-exp
//                                   mode also keeps E = exp(z - r) in bf16, r the row's
//                                   reference logit (teacher kernel)
//     combine                       lse_t, l_t, gradient multipliers
//     stored-exp mode:  repair      rows whose stored exps used a per-tile reference
//                                   rescaled to the row's reference R (usually none)
//     recompute mode:   GRAD        G = (mask/N) M exp(z - lse), z formed again
//     fixup                         G at the K ids: subtract (mask/N) P (stored-exp mode:
//                                   P / (M exp(R - lse)), as G = c_t E there), in place
//     DH contraction                split partials of G W (stored-exp: E W, and Hs = c_t H_c
//                                   from the epilogue warps before their first tile)
//       + teacher of chunk c + 1    launched behind it as a dependent (bf16 backward)
//     DW contraction                dW (+)= G^T H_c   (stored-exp: E^T Hs; TMA reduce-add)
//       + dH reduce                 dH_c = sum of the partials (stored-exp: times c_t),
//                                   launched behind it as a dependent
//   loss_finalize                   loss = sum mask l / N
// The gradient buffer G is the only one that grows with V, and it is bounded by
// chunk x V; everything else is O(T) or O(chunk x K).
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/ckl.h"
#include "common.cuh"
#include "kernels.h"

using namespace ckl;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct ProfRec {
  int kernel;
  int ev;
  double flops, bytes;
};

enum KernelId {
  KID_MASK = 0, KID_GATHER, KID_LSE, KID_COMBINE, KID_GRAD, KID_REPAIR, KID_FIXUP, KID_DH,
  KID_DW, KID_LOSS, KID_TKMAX, KID_TKTHRESH, KID_TKEMIT, KID_TKSELECT, KID_VP_MERGE,
  KID_DH_F32, KID_TO_BF16, KID_VP_GATHER, KID_VP_REDUCE, KID_COUNT
};
// bf16 backward: a profiled "dh_gemm" range also holds the next chunk's teacher
// kernel, and a "dw_gemm" range the chunk's dH split reduction, both launched
// behind the contraction as dependents (no event may stand between the two).
const char* kKernelNames[KID_COUNT] = {"mask_count", "teacher_topk", "lse_gemm", "lse_combine",
                                       "grad_gemm", "row_repair", "topk_fixup", "dh_gemm",
                                       "dw_gemm", "loss_finalize", "cache_max_gemm",
                                       "cache_threshold", "cache_emit_gemm", "cache_select",
                                       "vp_merge", "dh_reduce_f32", "dh_to_bf16",
                                       "vp_all_gather", "vp_all_reduce"};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

struct ckl_ctx {
  int device = 0;
  ckl_dtype dtype = CKL_F32;
  int64_t V = 0, d = 0, K = 0, max_chunk = 0;
  int num_sms = 0;
  unsigned* d_status = nullptr;  // device status word
  unsigned* h_status = nullptr;  // pinned
  float* h_loss = nullptr;       // pinned
  int64_t launches = 0;
  int recompute = 0;  // bf16: form the logits again in the backward (1) or keep exp(z) (0)
  EncodeTiledFn encode = nullptr;
  // profiling
  bool prof = false;
  std::vector<cudaEvent_t> ev;  // pairs: ev[2i], ev[2i+1]
  int ev_used = 0;
  std::vector<ProfRec> recs;
  // host-input calls: inputs are copied chunk by chunk on their own stream
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t copy_start = nullptr;
  std::vector<cudaEvent_t> chunk_ready;
};

namespace {

struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) return;
    ok = (prev == dev) || cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

struct WsPlan {
  int64_t Tc = 0;  // chunk rows planned for
  int n_vt = 0;    // vocabulary tiles of the log-sum-exp partials
  int64_t ldG = 0;
  int n_split = 1; // dH contraction splits (bf16)
  size_t off_ell = 0, off_lse = 0, off_misc = 0, off_tok = 0, off_cst = 0, off_zk = 0,
         off_Pk = 0, off_part = 0, off_xpart = 0, off_sid = 0, off_sp = 0, off_G = 0, off_dHp = 0,
         off_rep = 0, off_Hs = 0, total = 0;
  // vocabulary split over ranks: this rank's stats, the gathered stats, dH_c in fp32
  size_t off_stats = 0, off_stats_all = 0, off_dhf = 0;
};

// dH tiles are 256 x tc_bn(DH) outputs computed by CTA pairs; split the vocabulary
// (the contraction) so that the tile count fills the pairs evenly.
int pick_dh_split(int64_t Tc, int64_t d, int64_t V, int num_sms) {
  const int tw = tc_bn(TcKind::DH);
  const int64_t tiles = ((Tc + 255) / 256) * ((d + tw - 1) / tw);
  const int64_t n_kb = (V + 63) / 64;
  const int units = std::max(1, num_sms / 2);
  int best = 1;
  double best_cost = 1e300;
  for (int s = 1; s <= 8 && s <= n_kb; ++s) {
    const double waves = std::ceil((double)(tiles * s) / units);
    const double cost = waves / s + 0.01 * s;  // time per unit of tile work, plus partial traffic
    if (cost < best_cost - 1e-9) { best_cost = cost; best = s; }
  }
  // Every split must own at least one 64-wide block of the vocabulary.
  const int64_t kps = (n_kb + best - 1) / best;
  return (int)((n_kb + kps - 1) / kps);
}

WsPlan plan(const ckl_ctx* h, int64_t T, int64_t chunk, bool backward, int world = 0) {
  WsPlan p;
  p.Tc = std::max<int64_t>(1, std::min(chunk, std::max<int64_t>(T, 1)));
  const bool bf16 = h->dtype == CKL_BF16;
  p.n_vt = (int)((h->V + (bf16 ? 255 : 63)) / (bf16 ? 256 : 64));
  p.ldG = (int64_t)align_up((size_t)h->V, 8);
  p.n_split = bf16 ? pick_dh_split(p.Tc, h->d, h->V, h->num_sms) : 1;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  p.off_misc = take(sizeof(Misc));
  p.off_ell = take((size_t)std::max<int64_t>(T, 1) * 4);
  p.off_lse = take((size_t)std::max<int64_t>(T, 1) * 4);
  p.off_tok = take((size_t)p.Tc * 16);
  p.off_cst = take((size_t)p.Tc * 16);
  p.off_Pk = take((size_t)p.Tc * h->K * 4);
  p.off_part = take((size_t)p.n_vt * p.Tc * 8);
  if (bf16) {
    p.off_xpart = take((size_t)p.n_vt * p.Tc * 4);
    p.off_sid = take((size_t)p.Tc * h->K * 4);
    p.off_sp = take((size_t)p.Tc * h->K * 4);
  } else {
    p.off_zk = take((size_t)p.Tc * h->K * 4);
  }
  if (backward) {
    // bf16: blocked, 64 x 64 element blocks (8 KB); fp32: row-major, ldG
    p.off_G = bf16 ? take((size_t)((p.Tc + 63) / 64) * ((h->V + 63) / 64) * 8192)
                   : take((size_t)p.Tc * p.ldG * 4);
    if (bf16) {
      p.off_dHp = take((size_t)p.n_split * p.Tc * h->d * 4);
      // stored-exp backward: the repair list (count, rows) and the scaled H_c of DW
      p.off_rep = take((size_t)(p.Tc + 1) * 4);
      p.off_Hs = take((size_t)p.Tc * h->d * 2);
    }
  }
  if (world > 0) {
    p.off_stats = take((size_t)p.Tc * 16);
    p.off_stats_all = take((size_t)world * p.Tc * 16);
    p.off_dhf = take((size_t)p.Tc * h->d * 4);
  }
  p.total = o;
  return p;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// 2-D tensor map (bf16, or fp32 when f32 is set): `inner` contiguous elements per
// row, `outer` rows `row_bytes` apart, box of box_inner x box_outer, 128-byte
// swizzle, zero fill outside the tensor (loads) / clipping (stores).
// The bf16 gradient buffer of Tc tokens: 64 x 64 element blocks, 64 vocabulary ids
// fastest inside a block, then 64 tokens; blocks vocabulary-block-major within a
// token block. As a 4-D tensor (64, 64, vocabulary blocks, token blocks) with a
// box of 64 ids x box_t tokens x box_vb vocabulary blocks x box_tb token blocks.
bool make_map_g(const ckl_ctx* h, CUtensorMap* m, const void* base, int64_t V, int64_t Tc,
                uint32_t box_t, uint32_t box_vb, uint32_t box_tb) {
  const cuuint64_t n_vb = (cuuint64_t)((V + 63) / 64), n_tb = (cuuint64_t)((Tc + 63) / 64);
  const cuuint64_t dims[4] = {64, 64, n_vb, n_tb};
  const cuuint64_t strides[3] = {128, 8192, n_vb * 8192};
  const cuuint32_t box[4] = {64, box_t, box_vb, box_tb};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = h->encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base),
                               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map(const ckl_ctx* h, CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool f32 = false) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = h->encode(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                               2, const_cast<void*>(base),
                               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Every launch (and every caller-supplied collective) is wrapped in an NVTX range
// named after its kernel, so a timeline tool shows the call's structure; with no
// tool attached a range costs a few nanoseconds.
struct Launcher {
  ckl_ctx* h;
  cudaStream_t s;
  template <class F>
  cudaError_t operator()(int kid, double flops, double bytes, F&& f) {
    struct Range {
      explicit Range(const char* n) { nvtxRangePushA(n); }
      ~Range() { nvtxRangePop(); }
    } range(kKernelNames[kid]);
    int slot = -1;
    if (h->prof && h->ev_used * 2 + 1 < (int)h->ev.size()) {
      slot = h->ev_used++;
      cudaEventRecord(h->ev[2 * slot], s);
    }
    f();
    cudaError_t e = cudaGetLastError();
    if (slot >= 0) {
      cudaEventRecord(h->ev[2 * slot + 1], s);
      h->recs.push_back(ProfRec{kid, slot, flops, bytes});
    }
    h->launches++;
    return e;
  }
  // A caller-supplied collective: profiled under `kid`, not counted as a launch.
  template <class F>
  int collective(int kid, double bytes, F&& f) {
    nvtxRangePushA(kKernelNames[kid]);
    struct Pop {
      ~Pop() { nvtxRangePop(); }
    } pop;
    int slot = -1;
    if (h->prof && h->ev_used * 2 + 1 < (int)h->ev.size()) {
      slot = h->ev_used++;
      cudaEventRecord(h->ev[2 * slot], s);
    }
    const int rc = f();
    if (slot >= 0) {
      cudaEventRecord(h->ev[2 * slot + 1], s);
      h->recs.push_back(ProfRec{kid, slot, 0.0, bytes});
    }
    return rc;
  }
};

ckl_status check_common(const ckl_ctx* h, const void* H, const void* W, const int32_t* idx,
                        const float* logit, int64_t T, int64_t chunk, const float* loss) {
  if (!h) return CKL_ERR_INVALID_ARG;
  if (T < 0 || chunk < 1 || chunk > h->max_chunk || chunk > INT32_MAX) return CKL_ERR_INVALID_ARG;
  if (!W || !loss) return CKL_ERR_INVALID_ARG;
  if (T > 0 && (!H || !idx || !logit)) return CKL_ERR_INVALID_ARG;
  if (!aligned(W, 16) || (H && !aligned(H, 16)) || (idx && !aligned(idx, 16)) ||
      (logit && !aligned(logit, 16)) || !aligned(loss, 4))
    return CKL_ERR_ALIGNMENT;
  return CKL_OK;
}

// `group` (vocabulary split over ranks, bf16 only) or nullptr. `ready` (or
// nullptr): one event per chunk, recorded once that chunk's inputs (and, for
// chunk 0, the mask) are on the device; the stream waits for it before using them.
ckl_status run(ckl_ctx* h, const void* H, const void* W, const int32_t* idx, const float* logit,
               const uint8_t* mask, int64_t T, int64_t chunk, float* loss, void* dH, float* dW,
               float* tok_lse, float* tok_loss, void* ws, size_t ws_bytes, cudaStream_t s,
               bool backward, const ckl_vocab_group* group = nullptr,
               const cudaEvent_t* ready = nullptr) {
  ckl_status st = check_common(h, H, W, idx, logit, T, chunk, loss);
  if (st != CKL_OK) return st;
  if (backward) {
    if (!dW || (T > 0 && !dH)) return CKL_ERR_INVALID_ARG;
    if (!aligned(dW, 16) || (dH && !aligned(dH, 16))) return CKL_ERR_ALIGNMENT;
  }
  if ((tok_lse && !aligned(tok_lse, 4)) || (tok_loss && !aligned(tok_loss, 4)))
    return CKL_ERR_ALIGNMENT;
  const WsPlan P = plan(h, T, chunk, backward, group ? group->world : 0);
  if (!ws || !aligned(ws, 256) || ws_bytes < P.total) return CKL_ERR_WORKSPACE;

  DeviceGuard guard(h->device);
  if (!guard.ok) return CKL_ERR_CUDA;
  cudaGetLastError();  // clear a stale error so that launch checks below are ours

  unsigned char* base = static_cast<unsigned char*>(ws);
  ChunkBufs b;
  b.misc = reinterpret_cast<Misc*>(base + P.off_misc);
  b.tok = reinterpret_cast<float4*>(base + P.off_tok);
  b.cst = reinterpret_cast<float4*>(base + P.off_cst);
  b.zk = h->dtype == CKL_BF16 ? nullptr : reinterpret_cast<float*>(base + P.off_zk);
  b.Pk = reinterpret_cast<float*>(base + P.off_Pk);
  b.part = reinterpret_cast<float2*>(base + P.off_part);
  b.xpart = h->dtype == CKL_BF16 ? reinterpret_cast<float*>(base + P.off_xpart) : nullptr;
  b.sid = h->dtype == CKL_BF16 ? reinterpret_cast<int32_t*>(base + P.off_sid) : nullptr;
  b.sp = h->dtype == CKL_BF16 ? reinterpret_cast<float*>(base + P.off_sp) : nullptr;
  b.G = backward ? base + P.off_G : nullptr;
  b.dHp = (backward && h->dtype == CKL_BF16) ? reinterpret_cast<float*>(base + P.off_dHp) : nullptr;
  b.rep = (backward && h->dtype == CKL_BF16) ? reinterpret_cast<int*>(base + P.off_rep) : nullptr;
  uint16_t* Hs = (backward && h->dtype == CKL_BF16) ? reinterpret_cast<uint16_t*>(base + P.off_Hs)
                                                     : nullptr;
  float* ell_all = reinterpret_cast<float*>(base + P.off_ell);
  float* lse_all = reinterpret_cast<float*>(base + P.off_lse);
  float4* stats = group ? reinterpret_cast<float4*>(base + P.off_stats) : nullptr;
  float4* stats_all = group ? reinterpret_cast<float4*>(base + P.off_stats_all) : nullptr;
  float* dhf = group ? reinterpret_cast<float*>(base + P.off_dhf) : nullptr;
  const int V_all = group ? (int)group->V_total : (int)h->V;
  const int v0 = group ? (int)group->v0 : 0;
  int coll_rc = 0;          // first failing collective's return code
  bool map_failed = false;  // a tensor map could not be encoded

  const int V = (int)h->V, d = (int)h->d, K = (int)h->K;
  const bool bf16 = h->dtype == CKL_BF16;
  const size_t esz = bf16 ? 2 : 4;
  Launcher L{h, s};
  cudaError_t err = cudaSuccess;
  auto chk = [&](cudaError_t e) { if (e != cudaSuccess && err == cudaSuccess) err = e; };

  if (ready && T > 0) chk(cudaStreamWaitEvent(s, ready[0], 0));
  chk(L(KID_MASK, 0, (double)T, [&] { launch_mask_count(mask, T, b.misc, s); }));
  if (backward && T == 0) chk(cudaMemsetAsync(dW, 0, (size_t)V * d * 4, s));

  // bf16 backward: each chunk after the first has its teacher kernel launched behind
  // the previous chunk's dH contraction, which it overlaps (it reads only that
  // chunk's inputs and writes only per-chunk buffers the previous chunk no longer
  // reads once its dH contraction starts).
  bool teacher_queued = false;
  // With a group every chunk makes its two collectives even after an error (the
  // ranks' calls must stay matched); only the kernels are skipped.
  for (int64_t t0 = 0; t0 < T && (err == cudaSuccess || group); t0 += chunk) {
    const int Tc = (int)std::min<int64_t>(chunk, T - t0);
    const double zflops = 2.0 * Tc * (double)V * d;
    const unsigned char* Hc = static_cast<const unsigned char*>(H) + (size_t)t0 * d * esz;
    // The chunk's collectives (group only): one all-gather, and with a backward
    // one all-reduce. `drain` makes those not made yet, after a failure.
    bool gathered = false, reduced = false;
    auto gather = [&] {
      gathered = true;
      if (coll_rc) return;
      coll_rc = L.collective(KID_VP_GATHER, (double)group->world * Tc * 16, [&] {
        return group->all_gather(group->user, reinterpret_cast<const float*>(stats),
                                 reinterpret_cast<float*>(stats_all), (int64_t)Tc * 4, s);
      });
    };
    auto reduce = [&] {
      reduced = true;
      if (coll_rc || !backward) return;
      coll_rc = L.collective(KID_VP_REDUCE, (double)Tc * d * 4, [&] {
        return group->all_reduce_sum(group->user, dhf, (int64_t)Tc * d, s);
      });
    };
    auto drain = [&] {
      if (!group) return;
      if (!gathered) gather();
      if (!reduced) reduce();
    };
    if (err != cudaSuccess || coll_rc != 0 || map_failed) {
      drain();
      continue;
    }
    if (ready) chk(cudaStreamWaitEvent(s, ready[t0 / chunk], 0));

    // bf16 backward keeps the exps of the forward contraction (unless recomputing)
    const bool store_e = bf16 && backward && !h->recompute;
    if (bf16 && !teacher_queued) {
      chk(L(KID_GATHER, 0, (double)Tc * K * 16.0 + (store_e ? 4.0 * Tc * d : 0.0), [&] {
        launch_teacher(idx, logit, t0, Tc, V_all, v0, V, K, b, h->d_status,
                       store_e ? reinterpret_cast<const uint16_t*>(Hc) : nullptr,
                       static_cast<const uint16_t*>(W), d, false, s);
      }));
    } else if (bf16) {
      teacher_queued = false;  // launched behind the previous chunk's dH contraction
    } else {
      chk(L(KID_GATHER, 2.0 * Tc * K * d, (double)Tc * (K * 8.0 + d * esz + K * d * esz), [&] {
        launch_gather<float>(static_cast<const float*>(H), static_cast<const float*>(W), idx,
                             logit, t0, Tc, d, V, K, b, h->d_status, s);
      }));
    }

    // bf16: z = H_c W^T on the tensor cores. Stored-exp mode also writes
    // exp(z - row reference) into the gradient buffer (map c) for the backward.
    TcMaps mz;
    if (bf16) {
      if (!make_map(h, &mz.a, Hc, d, Tc, (uint64_t)d * 2, 64, 128) ||
          !make_map(h, &mz.b, W, d, V, (uint64_t)d * 2, 64, 128) ||
          (backward && !make_map_g(h, &mz.c, b.G, V, Tc, 32, 1, 1))) {
        map_failed = true;
        if (!group) return CKL_ERR_CUDA;
        drain();
        continue;
      }
      if (!backward) mz.c = mz.a;
    }
    chk(L(KID_LSE, zflops, store_e ? (double)Tc * V * 2 : 0, [&] {
      if (bf16) {
        TcLaunch p{};
        p.kind = TcKind::LSE; p.M = Tc; p.N = V; p.n_kb = (d + 63) / 64; p.n_split = 1; p.V = V;
        p.part = b.part; p.part_ld = Tc; p.store_e = store_e ? 1 : 0;
        p.sid = b.sid; p.sp = b.sp; p.xpart = b.xpart; p.K = K; p.tok = b.tok;
        p.status = h->d_status; p.num_sms = h->num_sms;
        launch_tc(mz, p, s);
      } else {
        launch_simt_lse(reinterpret_cast<const float*>(Hc), static_cast<const float*>(W), Tc, V,
                        d, b.part, s);
      }
    }));
    chk(L(KID_COMBINE, 0, (double)P.n_vt * Tc * 8, [&] {
      launch_combine(t0, Tc, P.n_vt, mask, b, lse_all, ell_all, stats, store_e, s);
    }));
    if (group) {
      // this rank's (max, sum, cross) per token to every rank; merged in rank order
      gather();
      chk(L(KID_VP_MERGE, 0, (double)Tc * (group->world * 16.0 + 24.0), [&] {
        launch_vp_merge(t0, Tc, group->world, group->rank, stats_all, mask, b, lse_all, ell_all,
                        store_e, s);
      }));
    }
    if (!backward) continue;

    if (store_e) {
      chk(L(KID_REPAIR, 0, 0, [&] {
        launch_repair(static_cast<uint16_t*>(b.G), Tc, V, b, h->num_sms, s);
      }));
    } else {
      chk(L(KID_GRAD, zflops, (double)Tc * V * esz, [&] {
        if (bf16) {
          TcLaunch p{};
          p.kind = TcKind::GRAD; p.M = Tc; p.N = V; p.n_kb = (d + 63) / 64; p.n_split = 1; p.V = V;
          p.cst = b.cst; p.G = static_cast<uint16_t*>(b.G); p.ldG = P.ldG;
          p.status = h->d_status; p.num_sms = h->num_sms;
          launch_tc(mz, p, s);
        } else {
          launch_simt_grad(reinterpret_cast<const float*>(Hc), static_cast<const float*>(W), Tc,
                           V, d, b.cst, static_cast<float*>(b.G), P.ldG, s);
        }
      }));
    }
    chk(L(KID_FIXUP, 0, (double)Tc * K * (12.0 + 2 * esz), [&] {
      if (bf16) launch_fixup<uint16_t>(idx, t0, Tc, K, V, v0, (V + 63) / 64, b, store_e, s);
      else launch_fixup<float>(idx, t0, Tc, K, V, v0, P.ldG, b, false, s);
    }));

    unsigned char* dHc = static_cast<unsigned char*>(dH) + (size_t)t0 * d * esz;
    if (bf16) {
      TcMaps mh, mw;
      if (!make_map_g(h, &mh.a, b.G, V, Tc, 64, 1, 2) ||
          !make_map(h, &mh.b, W, d, V, (uint64_t)d * 2, 64, 64) ||
          !make_map_g(h, &mw.a, b.G, V, Tc, 64, 2, 1) ||
          !make_map(h, &mw.b, store_e ? static_cast<const void*>(Hs) : Hc, d, Tc,
                    (uint64_t)d * 2, 64, 64) ||
          !make_map(h, &mw.c, dW, d, V, (uint64_t)d * 4, 32, 32, true)) {
        map_failed = true;
        if (!group) return CKL_ERR_CUDA;
        drain();
        continue;
      }
      mh.c = mh.a;
      // The next chunk's teacher kernel goes behind this dH contraction (its inputs
      // must be on the device first).
      const int64_t t1 = t0 + chunk;
      const int Tc1 = (int)std::min<int64_t>(chunk, T - t1);
      const bool queue_next = t1 < T && err == cudaSuccess;
      if (queue_next && ready) chk(cudaStreamWaitEvent(s, ready[t1 / chunk], 0));
      chk(L(KID_DH, zflops, 0, [&] {
        TcLaunch p{};
        p.kind = TcKind::DH; p.M = Tc; p.N = d; p.n_kb = (V + 63) / 64; p.n_split = P.n_split;
        p.dHp = b.dHp; p.status = h->d_status; p.num_sms = h->num_sms;
        if (store_e) {
          p.cst = b.cst;
          p.Hc = reinterpret_cast<const uint16_t*>(Hc);
          p.Hs = Hs;
        }
        launch_tc(mh, p, s);
        if (queue_next) {
          // timed, when profiling, inside this record: nothing may stand between the two
          const unsigned char* H1 = static_cast<const unsigned char*>(H) + (size_t)t1 * d * esz;
          launch_teacher(idx, logit, t1, Tc1, V_all, v0, V, K, b, h->d_status,
                         store_e ? reinterpret_cast<const uint16_t*>(H1) : nullptr,
                         static_cast<const uint16_t*>(W), d, true, s);
          h->launches++;
          teacher_queued = true;
        }
      }));
      if (group) {
        // this rank's share of dH_c in fp32, summed over ranks, then bf16
        chk(L(KID_DH_F32, 0, (double)Tc * d * (4.0 * P.n_split + 4.0), [&] {
          launch_dh_reduce_f32(b.dHp, P.n_split, (int64_t)Tc * d, dhf, d,
                               store_e ? b.cst : nullptr, s);
        }));
        reduce();
        chk(L(KID_TO_BF16, 0, (double)Tc * d * 6.0, [&] {
          launch_f32_to_bf16(dhf, (int64_t)Tc * d, reinterpret_cast<uint16_t*>(dHc), s);
        }));
      }
      chk(L(KID_DW, zflops, 0, [&] {
        TcLaunch p{};
        p.kind = TcKind::DW; p.M = V; p.N = d; p.n_kb = (Tc + 63) / 64; p.n_split = 1;
        p.dW = dW; p.first = t0 == 0; p.status = h->d_status; p.num_sms = h->num_sms;
        launch_tc(mw, p, s);
        if (!group) {
          // dH_c's split reduction behind the dW contraction, in the same record
          launch_dh_reduce_bf16(b.dHp, P.n_split, (int64_t)Tc * d,
                                reinterpret_cast<uint16_t*>(dHc), d, store_e ? b.cst : nullptr,
                                h->num_sms, s);
          h->launches++;
        }
      }));
    } else {
      const float* G = static_cast<const float*>(b.G);
      chk(L(KID_DH, zflops, 0, [&] {
        launch_simt_gemm(G, P.ldG, 1, static_cast<const float*>(W), 1, d,
                         reinterpret_cast<float*>(dHc), d, Tc, d, V, 0, s);
      }));
      chk(L(KID_DW, zflops, 0, [&] {
        launch_simt_gemm(G, 1, P.ldG, reinterpret_cast<const float*>(Hc), 1, d, dW, d, V, d, Tc,
                         t0 > 0, s);
      }));
    }
  }
  chk(L(KID_LOSS, 0, (double)T * 5, [&] { launch_loss_finalize(ell_all, mask, T, b.misc, loss, s); }));
  if (T > 0 && tok_lse)
    chk(cudaMemcpyAsync(tok_lse, lse_all, (size_t)T * 4, cudaMemcpyDeviceToDevice, s));
  if (T > 0 && tok_loss)
    chk(cudaMemcpyAsync(tok_loss, ell_all, (size_t)T * 4, cudaMemcpyDeviceToDevice, s));
  if (err != cudaSuccess) {
    std::fprintf(stderr, "ckl: CUDA error: %s\n", cudaGetErrorString(err));
    return CKL_ERR_CUDA;
  }
  if (map_failed) return CKL_ERR_CUDA;
  if (coll_rc != 0) return CKL_ERR_COLLECTIVE;
  return CKL_OK;
}

// Workspace of the teacher top-K cache builder for one chunk of Tc rows.
struct TopkPlan {
  int64_t Tc = 0;
  int n_vt = 0;  // 256-wide vocabulary tiles
  int cap = 0;   // candidates per row: at most K tiles can beat the threshold
  size_t off_tbest = 0, off_theta = 0, off_cnt = 0, off_cand = 0, total = 0;
  // vocabulary split over ranks: this rank's K best, packed, gathered, regrouped
  size_t off_loc_idx = 0, off_loc_lg = 0, off_packed = 0, off_gathered = 0, off_cand2 = 0,
         off_cnt2 = 0;
};

TopkPlan topk_plan(const ckl_ctx* h, int64_t T, int64_t chunk, int world = 0) {
  TopkPlan p;
  p.Tc = std::max<int64_t>(1, std::min(chunk, std::max<int64_t>(T, 1)));
  p.n_vt = (int)((h->V + 255) / 256);
  p.cap = (int)std::min<int64_t>(h->V, h->K * 256);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  p.off_tbest = take((size_t)p.n_vt * p.Tc * 8);
  p.off_theta = take((size_t)p.Tc * 8);
  p.off_cnt = take((size_t)p.Tc * 4);
  p.off_cand = take((size_t)p.Tc * p.cap * 8);
  if (world > 0) {
    const size_t tk = (size_t)p.Tc * h->K;
    p.off_loc_idx = take(tk * 4);
    p.off_loc_lg = take(tk * 4);
    p.off_packed = take(tk * 8);
    p.off_gathered = take(tk * 8 * world);
    p.off_cand2 = take(tk * 8 * world);
    p.off_cnt2 = take((size_t)p.Tc * 4);
  }
  p.total = o;
  return p;
}

ckl_status fold_status(unsigned dev) {
  if (dev & ST_INDEX_RANGE) return CKL_ERR_INDEX_RANGE;
  if (dev & ST_TIMEOUT) return CKL_ERR_TIMEOUT;
  if (dev & ST_INTERNAL) return CKL_ERR_INTERNAL;
  return CKL_OK;
}

// Copy the loss and the device status to pinned host memory, wait, clear the
// status word.
ckl_status sync_and_read(ckl_ctx* h, cudaStream_t s, const float* loss_dev, float* loss_host) {
  if (loss_dev && cudaMemcpyAsync(h->h_loss, loss_dev, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return CKL_ERR_CUDA;
  if (cudaMemcpyAsync(h->h_status, h->d_status, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemsetAsync(h->d_status, 0, 4, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
    return CKL_ERR_CUDA;
  if (loss_host && loss_dev) *loss_host = *h->h_loss;
  return fold_status(*h->h_status);
}

}  // namespace

extern "C" {

const char* ckl_status_str(ckl_status s) {
  switch (s) {
    case CKL_OK: return "ok";
    case CKL_ERR_INVALID_ARG: return "invalid argument";
    case CKL_ERR_UNSUPPORTED: return "unsupported size";
    case CKL_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case CKL_ERR_INDEX_RANGE: return "a top-K index is outside [0, V)";
    case CKL_ERR_CUDA: return "CUDA runtime error";
    case CKL_ERR_TIMEOUT: return "device pipeline wait timed out";
    case CKL_ERR_ALIGNMENT: return "pointer misaligned";
    case CKL_ERR_INTERNAL: return "internal consistency check failed";
    case CKL_ERR_COLLECTIVE: return "a caller-supplied collective failed";
  }
  return "unknown status";
}

ckl_status ckl_create(ckl_handle* out, int device, ckl_dtype dtype, int64_t V, int64_t d,
                      int64_t K, int64_t max_chunk) {
  if (!out) return CKL_ERR_INVALID_ARG;
  *out = nullptr;
  if (dtype != CKL_F32 && dtype != CKL_BF16) return CKL_ERR_INVALID_ARG;
  if (V < 1 || d < 1 || K < 1 || max_chunk < 1 || device < 0) return CKL_ERR_INVALID_ARG;
  if (d % 8 != 0 || K > 1024 || V > (int64_t)INT32_MAX / 2 || d > 65536 || max_chunk > INT32_MAX)
    return CKL_ERR_UNSUPPORTED;
  const int64_t per_warp = ((d * (dtype == CKL_BF16 ? 2 : 4) + 15) / 16) * 16 + 2 * ((K * 4 + 15) / 16) * 16;
  if (4 * per_warp > 200 * 1024) return CKL_ERR_UNSUPPORTED;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device >= ndev) return CKL_ERR_CUDA;
  DeviceGuard guard(device);
  if (!guard.ok) return CKL_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return CKL_ERR_CUDA;
  if (dtype == CKL_BF16 && prop.major != 10) return CKL_ERR_UNSUPPORTED;  // tcgen05 kernels are sm_100a

  ckl_ctx* h = new ckl_ctx();
  h->device = device;
  h->dtype = dtype;
  h->V = V; h->d = d; h->K = K; h->max_chunk = max_chunk;
  h->num_sms = prop.multiProcessorCount;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn) {
    delete h;
    return CKL_ERR_CUDA;
  }
  h->encode = reinterpret_cast<EncodeTiledFn>(fn);
  if (cudaMalloc(&h->d_status, 16) != cudaSuccess) { delete h; return CKL_ERR_CUDA; }
  if (cudaMallocHost(&h->h_status, 16) != cudaSuccess) {
    cudaFree(h->d_status);
    delete h;
    return CKL_ERR_CUDA;
  }
  h->h_loss = reinterpret_cast<float*>(h->h_status + 1);
  cudaMemset(h->d_status, 0, 16);
  if (cudaDeviceSynchronize() != cudaSuccess) { ckl_destroy(h); return CKL_ERR_CUDA; }
  *out = h;
  return CKL_OK;
}

ckl_status ckl_destroy(ckl_handle h) {
  if (!h) return CKL_OK;
  DeviceGuard guard(h->device);
  for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
  for (cudaEvent_t e : h->chunk_ready) cudaEventDestroy(e);
  if (h->copy_start) cudaEventDestroy(h->copy_start);
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
  if (h->d_status) cudaFree(h->d_status);
  if (h->h_status) cudaFreeHost(h->h_status);
  delete h;
  return CKL_OK;
}

ckl_status ckl_workspace_bytes(ckl_handle h, int64_t T, int64_t chunk, size_t* bytes) {
  if (!h || !bytes || T < 0 || chunk < 1) return CKL_ERR_INVALID_ARG;
  *bytes = plan(h, T, chunk, true).total;
  return CKL_OK;
}

ckl_status ckl_fwd_bwd(ckl_handle h, const void* H, const void* W, const int32_t* topk_idx,
                       const float* topk_logit, const uint8_t* mask, int64_t T, int64_t chunk,
                       float* loss, void* dH, float* dW, float* token_lse, float* token_loss,
                       void* workspace, size_t workspace_bytes, void* stream, float* loss_host) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ckl_status st = run(h, H, W, topk_idx, topk_logit, mask, T, chunk, loss, dH, dW, token_lse,
                      token_loss, workspace, workspace_bytes, s, true);
  if (st != CKL_OK || !loss_host) return st;
  DeviceGuard guard(h->device);
  return sync_and_read(h, s, loss, loss_host);
}

ckl_status ckl_forward(ckl_handle h, const void* H, const void* W, const int32_t* topk_idx,
                       const float* topk_logit, const uint8_t* mask, int64_t T, int64_t chunk,
                       float* loss, float* token_lse, float* token_loss, void* workspace,
                       size_t workspace_bytes, void* stream, float* loss_host) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ckl_status st = run(h, H, W, topk_idx, topk_logit, mask, T, chunk, loss, nullptr, nullptr,
                      token_lse, token_loss, workspace, workspace_bytes, s, false);
  if (st != CKL_OK || !loss_host) return st;
  DeviceGuard guard(h->device);
  return sync_and_read(h, s, loss, loss_host);
}

ckl_status ckl_fwd_bwd_from_host(ckl_handle h, const void* H_host, const int32_t* idx_host,
                                 const float* logit_host, const uint8_t* mask_host, void* H_dev,
                                 int32_t* idx_dev, float* logit_dev, uint8_t* mask_dev,
                                 const void* W, int64_t T, int64_t chunk, float* loss, void* dH,
                                 float* dW, void* workspace, size_t workspace_bytes, void* stream,
                                 float* loss_host) {
  if (!h || !loss_host || T < 0 || chunk < 1) return CKL_ERR_INVALID_ARG;
  if (T > 0 && (!H_host || !idx_host || !logit_host || !H_dev || !idx_dev || !logit_dev))
    return CKL_ERR_INVALID_ARG;
  if (mask_host && !mask_dev) return CKL_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n_chunks = T > 0 ? (T + chunk - 1) / chunk : 0;
  {
    DeviceGuard guard(h->device);
    if (!guard.ok) return CKL_ERR_CUDA;
    // The inputs go up chunk by chunk on the handle's copy stream, so chunk c + 1
    // crosses the bus while chunk c computes. The copies start after everything
    // already enqueued on `stream` (which may still read these device buffers).
    if (!h->copy_stream &&
        (cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking) != cudaSuccess ||
         cudaEventCreateWithFlags(&h->copy_start, cudaEventDisableTiming) != cudaSuccess))
      return CKL_ERR_CUDA;
    while ((int64_t)h->chunk_ready.size() < n_chunks) {
      cudaEvent_t e;
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return CKL_ERR_CUDA;
      h->chunk_ready.push_back(e);
    }
    cudaStream_t c = h->copy_stream;
    if (cudaEventRecord(h->copy_start, s) != cudaSuccess ||
        cudaStreamWaitEvent(c, h->copy_start, 0) != cudaSuccess)
      return CKL_ERR_CUDA;
    const size_t esz = h->dtype == CKL_BF16 ? 2 : 4;
    if (T > 0 && mask_host &&
        cudaMemcpyAsync(mask_dev, mask_host, (size_t)T, cudaMemcpyHostToDevice, c) != cudaSuccess)
      return CKL_ERR_CUDA;
    for (int64_t k = 0; k < n_chunks; ++k) {
      const int64_t t0 = k * chunk, Tc = std::min<int64_t>(chunk, T - t0);
      const size_t hb = (size_t)h->d * esz, kb = (size_t)h->K * 4;
      if (cudaMemcpyAsync(static_cast<unsigned char*>(H_dev) + t0 * hb,
                          static_cast<const unsigned char*>(H_host) + t0 * hb, Tc * hb,
                          cudaMemcpyHostToDevice, c) != cudaSuccess ||
          cudaMemcpyAsync(idx_dev + t0 * h->K, idx_host + t0 * h->K, Tc * kb,
                          cudaMemcpyHostToDevice, c) != cudaSuccess ||
          cudaMemcpyAsync(logit_dev + t0 * h->K, logit_host + t0 * h->K, Tc * kb,
                          cudaMemcpyHostToDevice, c) != cudaSuccess ||
          cudaEventRecord(h->chunk_ready[k], c) != cudaSuccess)
        return CKL_ERR_CUDA;
    }
  }
  ckl_status st = run(h, H_dev, W, idx_dev, logit_dev, mask_host ? mask_dev : nullptr, T, chunk,
                      loss, dH, dW, nullptr, nullptr, workspace, workspace_bytes, s, true, nullptr,
                      n_chunks ? h->chunk_ready.data() : nullptr);
  if (st != CKL_OK) {
    // the copies may still be running: do not return while they read the caller's buffers
    DeviceGuard guard(h->device);
    cudaStreamSynchronize(h->copy_stream);
    return st;
  }
  DeviceGuard guard(h->device);
  return sync_and_read(h, s, loss, loss_host);
}

ckl_status ckl_vp_workspace_bytes(ckl_handle h, int32_t world, int64_t T, int64_t chunk,
                                  size_t* bytes) {
  if (!h || !bytes || world < 1 || T < 0 || chunk < 1) return CKL_ERR_INVALID_ARG;
  *bytes = plan(h, T, chunk, true, world).total;
  return CKL_OK;
}

namespace {
ckl_status check_group(const ckl_ctx* h, const ckl_vocab_group* g, bool backward) {
  if (!h || !g || g->world < 1 || g->rank < 0 || g->rank >= g->world || !g->all_gather ||
      (backward && !g->all_reduce_sum) || g->v0 < 0 || g->V_total > INT32_MAX ||
      g->v0 + h->V > g->V_total)
    return CKL_ERR_INVALID_ARG;
  if (h->dtype != CKL_BF16) return CKL_ERR_UNSUPPORTED;
  return CKL_OK;
}
}  // namespace

ckl_status ckl_forward_vocab_parallel(ckl_handle h, const ckl_vocab_group* g, const void* H,
                                      const void* W_shard, const int32_t* topk_idx,
                                      const float* topk_logit, const uint8_t* mask, int64_t T,
                                      int64_t chunk, float* loss, float* token_lse,
                                      float* token_loss, void* workspace, size_t workspace_bytes,
                                      void* stream, float* loss_host) {
  ckl_status st = check_group(h, g, false);
  if (st != CKL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = run(h, H, W_shard, topk_idx, topk_logit, mask, T, chunk, loss, nullptr, nullptr, token_lse,
           token_loss, workspace, workspace_bytes, s, false, g);
  if (st != CKL_OK || !loss_host) return st;
  DeviceGuard guard(h->device);
  return sync_and_read(h, s, loss, loss_host);
}

ckl_status ckl_fwd_bwd_vocab_parallel(ckl_handle h, const ckl_vocab_group* g, const void* H,
                                      const void* W_shard, const int32_t* topk_idx,
                                      const float* topk_logit, const uint8_t* mask, int64_t T,
                                      int64_t chunk, float* loss, void* dH, float* dW_shard,
                                      float* token_lse, float* token_loss, void* workspace,
                                      size_t workspace_bytes, void* stream, float* loss_host) {
  ckl_status st = check_group(h, g, true);
  if (st != CKL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = run(h, H, W_shard, topk_idx, topk_logit, mask, T, chunk, loss, dH, dW_shard,
                      token_lse, token_loss, workspace, workspace_bytes, s, true, g);
  if (st != CKL_OK || !loss_host) return st;
  DeviceGuard guard(h->device);
  return sync_and_read(h, s, loss, loss_host);
}

ckl_status ckl_selftest_wait_bound(ckl_handle h, void* stream, int64_t* cycles) {
  if (!h) return CKL_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return CKL_ERR_CUDA;
  cudaGetLastError();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // bytes 8..15 of the handle's 16-byte status block (device and pinned host)
  long long* d_cyc = reinterpret_cast<long long*>(reinterpret_cast<unsigned char*>(h->d_status) + 8);
  long long* h_cyc = reinterpret_cast<long long*>(reinterpret_cast<unsigned char*>(h->h_status) + 8);
  launch_wait_selftest(h->d_status, d_cyc, s);
  if (cudaGetLastError() != cudaSuccess) return CKL_ERR_CUDA;
  if (cudaMemcpyAsync(h_cyc, d_cyc, 8, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return CKL_ERR_CUDA;
  const ckl_status st = sync_and_read(h, s, nullptr, nullptr);
  if (cycles) *cycles = *h_cyc;
  return st;
}

ckl_status ckl_sync_status(ckl_handle h, void* stream) {
  if (!h) return CKL_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return CKL_ERR_CUDA;
  return sync_and_read(h, static_cast<cudaStream_t>(stream), nullptr, nullptr);
}

int64_t ckl_launch_count(ckl_handle h) { return h ? h->launches : -1; }

ckl_status ckl_topk_workspace_bytes(ckl_handle h, int64_t T, int64_t chunk, size_t* bytes) {
  if (!h || !bytes || T < 0 || chunk < 1) return CKL_ERR_INVALID_ARG;
  *bytes = topk_plan(h, T, chunk).total;
  return CKL_OK;
}

namespace {
// The cache builder. With `group` (vocabulary split over ranks) each rank builds
// the K best of its own rows into the extra buffers of the workspace, the pairs
// are all-gathered per chunk, and every rank selects the final K of the world * K
// candidates: the same result, bit for bit, as one rank holding all of W.
ckl_status topk_run(ckl_ctx* h, const ckl_vocab_group* group, const void* H, const void* W,
                    int64_t T, int64_t chunk, int32_t* topk_idx, float* topk_logit,
                    void* workspace, size_t workspace_bytes, void* stream, int wait) {
  if (!h || !W || T < 0 || chunk < 1 || chunk > h->max_chunk || chunk > INT32_MAX)
    return CKL_ERR_INVALID_ARG;
  if (T > 0 && (!H || !topk_idx || !topk_logit)) return CKL_ERR_INVALID_ARG;
  if (h->dtype != CKL_BF16 || h->K > h->V) return CKL_ERR_UNSUPPORTED;
  if (!aligned(W, 16) || (H && !aligned(H, 16)) || (topk_idx && !aligned(topk_idx, 4)) ||
      (topk_logit && !aligned(topk_logit, 4)))
    return CKL_ERR_ALIGNMENT;
  const TopkPlan P = topk_plan(h, T, chunk, group ? group->world : 0);
  if (T > 0 && (!workspace || !aligned(workspace, 256) || workspace_bytes < P.total))
    return CKL_ERR_WORKSPACE;
  DeviceGuard guard(h->device);
  if (!guard.ok) return CKL_ERR_CUDA;
  cudaGetLastError();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int V = (int)h->V, d = (int)h->d, K = (int)h->K;
  unsigned char* base = static_cast<unsigned char*>(workspace);
  float2* tbest = reinterpret_cast<float2*>(base + P.off_tbest);
  float2* theta = reinterpret_cast<float2*>(base + P.off_theta);
  int* cnt = reinterpret_cast<int*>(base + P.off_cnt);
  float2* cand = reinterpret_cast<float2*>(base + P.off_cand);
  int32_t* loc_idx = group ? reinterpret_cast<int32_t*>(base + P.off_loc_idx) : nullptr;
  float* loc_lg = group ? reinterpret_cast<float*>(base + P.off_loc_lg) : nullptr;
  float2* packed = group ? reinterpret_cast<float2*>(base + P.off_packed) : nullptr;
  float2* gathered = group ? reinterpret_cast<float2*>(base + P.off_gathered) : nullptr;
  float2* cand2 = group ? reinterpret_cast<float2*>(base + P.off_cand2) : nullptr;
  int* cnt2 = group ? reinterpret_cast<int*>(base + P.off_cnt2) : nullptr;
  Launcher L{h, s};
  cudaError_t err = cudaSuccess;
  int coll_rc = 0;
  bool map_failed = false;
  auto chk = [&](cudaError_t e) { if (e != cudaSuccess && err == cudaSuccess) err = e; };
  // With a group every chunk makes its one all-gather, also after a kernel
  // failure (the ranks' calls stay matched); only the kernels are skipped.
  for (int64_t t0 = 0; t0 < T && (err == cudaSuccess || group); t0 += chunk) {
    const int Tc = (int)std::min<int64_t>(chunk, T - t0);
    const double zflops = 2.0 * Tc * (double)V * d;
    const unsigned char* Hc = static_cast<const unsigned char*>(H) + (size_t)t0 * d * 2;
    auto gather = [&] {
      if (coll_rc) return;
      coll_rc = L.collective(KID_VP_GATHER, (double)group->world * Tc * K * 8, [&] {
        return group->all_gather(group->user, reinterpret_cast<const float*>(packed),
                                 reinterpret_cast<float*>(gathered), (int64_t)Tc * K * 2, s);
      });
    };
    if (err != cudaSuccess || coll_rc != 0 || map_failed) {
      gather();
      continue;
    }
    TcMaps m;
    if (!make_map(h, &m.a, Hc, d, Tc, (uint64_t)d * 2, 64, 128) ||
        !make_map(h, &m.b, W, d, V, (uint64_t)d * 2, 64, 128)) {
      map_failed = true;
      if (!group) return CKL_ERR_CUDA;
      gather();
      continue;
    }
    m.c = m.a;
    chk(cudaMemsetAsync(cnt, 0, (size_t)Tc * 4, s));
    chk(L(KID_TKMAX, zflops, 0, [&] {
      TcLaunch p{};
      p.kind = TcKind::TKMAX; p.M = Tc; p.N = V; p.n_kb = (d + 63) / 64; p.n_split = 1; p.V = V;
      p.part = tbest; p.part_ld = Tc; p.status = h->d_status; p.num_sms = h->num_sms;
      launch_tc(m, p, s);
    }));
    chk(L(KID_TKTHRESH, 0, (double)P.n_vt * Tc * 8, [&] {
      launch_topk_threshold(tbest, P.n_vt, Tc, K, theta, s);
    }));
    chk(L(KID_TKEMIT, zflops, 0, [&] {
      TcLaunch p{};
      p.kind = TcKind::TKEMIT; p.M = Tc; p.N = V; p.n_kb = (d + 63) / 64; p.n_split = 1; p.V = V;
      p.theta = theta; p.cand = cand; p.cand_cnt = cnt; p.cand_cap = P.cap;
      p.status = h->d_status; p.num_sms = h->num_sms;
      launch_tc(m, p, s);
    }));
    chk(L(KID_TKSELECT, 0, (double)Tc * K * 8, [&] {
      launch_topk_select(cand, cnt, P.cap, Tc, K, group ? loc_idx : topk_idx + t0 * K,
                         group ? loc_lg : topk_logit + t0 * K, h->d_status, s);
    }));
    if (group) {
      chk(L(KID_TKSELECT, 0, (double)Tc * K * 16, [&] {
        launch_topk_pack(loc_idx, loc_lg, (int64_t)Tc * K, (int)group->v0, packed, s);
      }));
      gather();
      chk(L(KID_TKSELECT, 0, (double)group->world * Tc * K * 16, [&] {
        launch_topk_regroup(gathered, group->world, Tc, K, cand2, cnt2, s);
      }));
      chk(L(KID_TKSELECT, 0, (double)group->world * Tc * K * 8, [&] {
        launch_topk_select(cand2, cnt2, group->world * K, Tc, K, topk_idx + t0 * K,
                           topk_logit + t0 * K, h->d_status, s);
      }));
    }
  }
  if (err != cudaSuccess) {
    std::fprintf(stderr, "ckl: CUDA error: %s\n", cudaGetErrorString(err));
    return CKL_ERR_CUDA;
  }
  if (map_failed) return CKL_ERR_CUDA;
  if (coll_rc != 0) return CKL_ERR_COLLECTIVE;
  if (!wait) return CKL_OK;
  return sync_and_read(h, s, nullptr, nullptr);
}
}  // namespace

ckl_status ckl_topk_cache(ckl_handle h, const void* H, const void* W, int64_t T, int64_t chunk,
                          int32_t* topk_idx, float* topk_logit, void* workspace,
                          size_t workspace_bytes, void* stream, int wait) {
  return topk_run(h, nullptr, H, W, T, chunk, topk_idx, topk_logit, workspace, workspace_bytes,
                  stream, wait);
}

ckl_status ckl_topk_vp_workspace_bytes(ckl_handle h, int32_t world, int64_t T, int64_t chunk,
                                       size_t* bytes) {
  if (!h || !bytes || world < 1 || T < 0 || chunk < 1) return CKL_ERR_INVALID_ARG;
  *bytes = topk_plan(h, T, chunk, world).total;
  return CKL_OK;
}

ckl_status ckl_topk_cache_vocab_parallel(ckl_handle h, const ckl_vocab_group* g, const void* H,
                                         const void* W_shard, int64_t T, int64_t chunk,
                                         int32_t* topk_idx, float* topk_logit, void* workspace,
                                         size_t workspace_bytes, void* stream, int wait) {
  if (!h || !g || g->world < 1 || g->rank < 0 || g->rank >= g->world || !g->all_gather ||
      g->v0 < 0 || g->V_total > INT32_MAX || g->v0 + h->V > g->V_total)
    return CKL_ERR_INVALID_ARG;
  return topk_run(h, g, H, W_shard, T, chunk, topk_idx, topk_logit, workspace, workspace_bytes,
                  stream, wait);
}

ckl_status ckl_set_recompute(ckl_handle h, int recompute) {
  if (!h) return CKL_ERR_INVALID_ARG;
  h->recompute = recompute != 0;
  return CKL_OK;
}

ckl_status ckl_profile_enable(ckl_handle h, int enable, int max_launches) {
  if (!h || max_launches < 0) return CKL_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return CKL_ERR_CUDA;
  h->prof = enable != 0;
  if (h->prof && (int)h->ev.size() < 2 * max_launches) {
    for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
    h->ev.assign(2 * (size_t)max_launches, nullptr);
    for (auto& e : h->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return CKL_ERR_CUDA;
  }
  h->ev_used = 0;
  h->recs.clear();
  return CKL_OK;
}

ckl_status ckl_profile_collect(ckl_handle h, ckl_kernel_stat* stats, int max_stats, int* n_stats) {
  if (!h || !n_stats || (max_stats > 0 && !stats)) return CKL_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return CKL_ERR_CUDA;
  ckl_kernel_stat acc[KID_COUNT];
  std::memset(acc, 0, sizeof(acc));
  for (const ProfRec& r : h->recs) {
    if (cudaEventSynchronize(h->ev[2 * r.ev + 1]) != cudaSuccess) return CKL_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, h->ev[2 * r.ev], h->ev[2 * r.ev + 1]) != cudaSuccess)
      return CKL_ERR_CUDA;
    ckl_kernel_stat& a = acc[r.kernel];
    a.launches++;
    a.total_ms += ms;
    a.flops += r.flops;
    a.bytes += r.bytes;
  }
  int n = 0;
  for (int k = 0; k < KID_COUNT; ++k) {
    if (acc[k].launches == 0) continue;
    if (n < max_stats) {
      stats[n] = acc[k];
      std::snprintf(stats[n].name, sizeof(stats[n].name), "%s", kKernelNames[k]);
    }
    ++n;
  }
  *n_stats = n;
  h->ev_used = 0;
  h->recs.clear();
  return CKL_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward-only loss without any device allocation.
//
// Some callers cannot call cudaMalloc: code embedded in a runtime that owns all
// device memory through its own arena or caching allocator (and forbids outside
// allocations), and latency-critical loops that cannot afford the device-wide
// synchronisation cudaMalloc / cudaFree imply. ckl_create allocates (a status
// word, a pinned host word), so this entry point takes no handle: its scratch
// (the status word plus the forward workspace) lives in one file-scope device
// array of kStaticScratchBytes that every GPU loading this library holds until
// the process exits. Calls share the array, so calls that overlap on the GPU
// (two streams, or two host threads) race and must be serialised by the caller.
namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr size_t kStaticStatusBytes = 256;                // status word, then the workspace
constexpr int kStaticMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

struct StaticDevice {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_static_scratch on this device
  int num_sms = 0;
  int cc_major = 0;
  EncodeTiledFn encode = nullptr;
};
std::mutex g_static_mu;
StaticDevice g_static_dev[kStaticMaxDevices];

// Once per device, with that device current: the device address of the static
// array (the host-side symbol is only a stand-in), the SM count and the TMA
// descriptor encoder. The address belongs to the device's current CUDA context;
// a cudaDeviceReset would end that context, which the header rules out.
ckl_status static_setup(int device, StaticDevice** out) {
  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticDevice& sd = g_static_dev[device];
  if (!sd.ready) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return CKL_ERR_CUDA;
    int sms = 0, major = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess)
      return CKL_ERR_CUDA;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return CKL_ERR_CUDA;
    sd.scratch = static_cast<unsigned char*>(ptr);
    sd.num_sms = sms;
    sd.cc_major = major;
    sd.encode = reinterpret_cast<EncodeTiledFn>(fn);
    sd.ready = true;
  }
  *out = &sd;
  return CKL_OK;
}

}  // namespace

extern "C" ckl_status ckl_forward_static(int device, ckl_dtype dtype, int64_t V, int64_t d,
                                         int64_t K, const void* H, const void* W,
                                         const int32_t* topk_idx, const float* topk_logit,
                                         const uint8_t* mask, int64_t T, int64_t chunk,
                                         float* loss, float* token_lse, float* token_loss,
                                         void* stream, float* loss_host) {
  if (dtype != CKL_F32 && dtype != CKL_BF16) return CKL_ERR_INVALID_ARG;
  if (V < 1 || d < 1 || K < 1 || chunk < 1 || T < 0 || device < 0 || device >= kStaticMaxDevices)
    return CKL_ERR_INVALID_ARG;
  // Without a handle the device status can only be returned by this call itself.
  if (!loss_host) return CKL_ERR_INVALID_ARG;
  if (d % 8 != 0 || K > 1024 || V > (int64_t)INT32_MAX / 2 || d > 65536 || chunk > INT32_MAX)
    return CKL_ERR_UNSUPPORTED;
  const int64_t per_warp =
      ((d * (dtype == CKL_BF16 ? 2 : 4) + 15) / 16) * 16 + 2 * ((K * 4 + 15) / 16) * 16;
  if (4 * per_warp > 200 * 1024) return CKL_ERR_UNSUPPORTED;
  DeviceGuard guard(device);
  if (!guard.ok) return CKL_ERR_CUDA;
  StaticDevice* sd = nullptr;
  ckl_status st = static_setup(device, &sd);
  if (st != CKL_OK) return st;
  if (dtype == CKL_BF16 && sd->cc_major != 10) return CKL_ERR_UNSUPPORTED;

  // A handle-shaped view of this call; it owns nothing.
  ckl_ctx c;
  c.device = device;
  c.dtype = dtype;
  c.V = V; c.d = d; c.K = K; c.max_chunk = chunk;
  c.num_sms = sd->num_sms;
  c.encode = sd->encode;
  c.d_status = reinterpret_cast<unsigned*>(sd->scratch);
  const WsPlan P = plan(&c, T, chunk, false);
  if (P.total > kStaticScratchBytes - kStaticStatusBytes) return CKL_ERR_WORKSPACE;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The status word must start at zero; every workspace piece the forward pass
  // reads is written earlier in the same call.
  if (cudaMemsetAsync(c.d_status, 0, sizeof(unsigned), s) != cudaSuccess) return CKL_ERR_CUDA;
  st = run(&c, H, W, topk_idx, topk_logit, mask, T, chunk, loss, nullptr, nullptr, token_lse,
           token_loss, sd->scratch + kStaticStatusBytes, kStaticScratchBytes - kStaticStatusBytes,
           s, false);
  if (st != CKL_OK) return st;
  unsigned dev_status = 0;
  float host_loss = 0.f;
  if (cudaMemcpyAsync(&host_loss, loss, sizeof(float), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(&dev_status, c.d_status, sizeof(unsigned), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return CKL_ERR_CUDA;
  *loss_host = host_loss;
  return fold_status(dev_status);
}
