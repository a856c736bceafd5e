// bf16 tensor-core contractions of the fused top-K forward-KL loss on sm_100a.
//
// One persistent, warp-specialised kernel template serves the four products of
// the method ("Chunked KL loss, running Knowledge Distillation locally in less
// <6GB VRAM", README "Full Chunked KL": the logits of a chunk exist only while
// the normaliser is being accumulated, and are formed a second time in the
// backward pass to build the analytic gradient):
//   LSE : z = H_c W^T tile by tile; the epilogue keeps only each row's
//         (max, sum of exp) over the tile's vocabulary columns.
//   GRAD: z recomputed; the epilogue writes G = gmul * exp(z - lse) in bf16.
//   DH  : dH_c = G W, contraction over the vocabulary split in n_split ranges
//         (fp32 partials, reduced in a fixed order afterwards).
//   DW  : dW (+)= G^T H_c, contraction over the chunk's tokens.
//
// CTA layout (192 threads, one CTA per SM):
//   warp 0      TMA producer: 128B-swizzled tiles of A and B into a STAGES-deep
//               shared-memory ring (mbarrier full/empty pairs).
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               (M=128, N=BN, K=16) into one of two TMEM accumulators and
//               commits each stage back to the producer.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (thread = output row),
//               then the kind's math and global stores, overlapped with the MMA
//               of the next tile through the second accumulator.
// Operand layouts: H, W and G are read K-major for LSE/GRAD/DH-A; W (DH-B), G
// (DW-A) and H (DW-B) are read MN-major, so no operand is ever transposed in
// memory. Every wait is bounded (common.cuh).
#include "common.cuh"
#include "kernels.h"

namespace ckl {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;               // 64 bf16 = one 128-byte swizzle row
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kAccStride = 256;      // TMEM columns between the two accumulators
constexpr int kAtomBytes = 64 * 128; // one 64 (MN) x 64 (K) MN-major box
constexpr float kLog2e = 1.4426950408889634f;

template <TcKind KIND>
struct Cfg;
template <> struct Cfg<TcKind::LSE>  { static constexpr int BN = 256; static constexpr bool A_MN = false, B_MN = false; static constexpr int STAGES = 4; };
template <> struct Cfg<TcKind::GRAD> { static constexpr int BN = 256; static constexpr bool A_MN = false, B_MN = false; static constexpr int STAGES = 4; };
template <> struct Cfg<TcKind::DH>   { static constexpr int BN = 192; static constexpr bool A_MN = false, B_MN = true;  static constexpr int STAGES = 5; };
template <> struct Cfg<TcKind::DW>   { static constexpr int BN = 192; static constexpr bool A_MN = true,  B_MN = true;  static constexpr int STAGES = 5; };

template <TcKind KIND>
struct Layout {
  static constexpr int BN = Cfg<KIND>::BN;
  static constexpr int STAGES = Cfg<KIND>::STAGES;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + RING_BYTES + BAR_BYTES;
};

struct TileCoord {
  int mt, nt, kb0, kb1, split;
};

__device__ __forceinline__ TileCoord tile_coord(const TcLaunch& p, int n_m, int n_n, int kps,
                                                int tile) {
  TileCoord c;
  c.split = 0;
  if (p.kind == TcKind::DW) {  // neighbouring CTAs share the A (gradient) tile
    c.nt = tile % n_n;
    c.mt = tile / n_n;
  } else {  // neighbouring CTAs share the B tile (W rows / columns)
    c.mt = tile % n_m;
    const int r = tile / n_m;
    c.nt = r % n_n;
    c.split = r / n_n;
  }
  c.kb0 = c.split * kps;
  c.kb1 = min(p.n_kb, c.kb0 + kps);
  return c;
}

template <TcKind KIND>
__global__ void __launch_bounds__(kThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const TcLaunch p) {
  using L = Layout<KIND>;
  constexpr int BN = L::BN;
  constexpr int STAGES = L::STAGES;
  constexpr bool A_MN = Cfg<KIND>::A_MN, B_MN = Cfg<KIND>::B_MN;

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::RING_BYTES);
  uint64_t* full = bars;                 // [STAGES]
  uint64_t* empty = bars + STAGES;       // [STAGES]
  uint64_t* tfull = bars + 2 * STAGES;   // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* done = tempty + 2;           // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_m = (p.M + BM - 1) / BM;
  const int n_n = (p.N + BN - 1) / BN;
  const int n_split = (KIND == TcKind::DH) ? p.n_split : 1;
  const int kps = (p.n_kb + n_split - 1) / n_split;
  const int n_tiles = n_m * n_n * n_split;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4 * 32);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_phase = 0;  // per-stage bits: loaded at least once / last parity
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
        const TileCoord c = tile_coord(p, n_m, n_n, kps, tile);
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          unsigned char* sA = smem + stage * L::STAGE_BYTES;
          unsigned char* sB = sA + L::A_BYTES;
          mbar_arrive_expect_tx(&full[stage], L::STAGE_BYTES);
          if (!A_MN) {
            tma_load_2d(sA, &tmA, &full[stage], kb * BK, c.mt * BM);
          } else {
#pragma unroll
            for (int a = 0; a < BM / 64; ++a)
              tma_load_2d(sA + a * kAtomBytes, &tmA, &full[stage], c.mt * BM + a * 64, kb * BK);
          }
          if (!B_MN) {
            tma_load_2d(sB, &tmB, &full[stage], kb * BK, c.nt * BN);
          } else {
#pragma unroll
            for (int a = 0; a < BN / 64; ++a)
              tma_load_2d(sB + a * kAtomBytes, &tmB, &full[stage], c.nt * BN + a * 64, kb * BK);
          }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Let every copy this thread issued land before the CTA can exit.
      for (int s = 0; s < STAGES; ++s) {
        if (!((issued >> s) & 1u)) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(&full[s], (issued_phase >> s) & 1u)) {
          if (clock64() - t0 > kWaitCycles) { atomicOr(p.status, (unsigned)ST_TIMEOUT); break; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++it) {
        const TileCoord c = tile_coord(p, n_m, n_n, kps, tile);
        const int buf = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * kAccStride);
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * L::STAGE_BYTES);
          const uint32_t b0 = a0 + L::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // K-major: step 16 elements (32 bytes) inside the 128-byte swizzle row.
            // MN-major: step 16 rows of 128 bytes; atoms along MN are kAtomBytes apart.
            const uint64_t ad = A_MN ? umma_desc_sw128(a0 + kk * 2048, kAtomBytes, 1024)
                                     : umma_desc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? umma_desc_sw128(b0 + kk * 2048, kAtomBytes, 1024)
                                     : umma_desc_sw128(b0 + kk * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (kb > c.kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[buf]);
      }
      // Every MMA issued above has completed once `done` flips.
      umma_commit(done);
      const long long t0 = clock64();
      while (!mbar_try_wait(done, 0)) {
        if (clock64() - t0 > kWaitCycles) { atomicOr(p.status, (unsigned)ST_TIMEOUT); break; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;   // accumulator row owned by this thread
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const TileCoord c = tile_coord(p, n_m, n_n, kps, tile);
      const int buf = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      if (!mbar_wait(&tfull[buf], use & 1u, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kAccStride);
      const int grow = c.mt * BM + row;  // output row (token for LSE/GRAD/DH, vocab id for DW)
      const bool row_ok = grow < p.M;
      const int col0 = c.nt * BN;

      if constexpr (KIND == TcKind::LSE) {
        float m2 = -INFINITY, s = 0.f;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          float v[32];
          tmem_ld32(taddr + cc * 32, v);
          const int cb = col0 + cc * 32;
          float cm = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            v[j] = (cb + j < p.V) ? v[j] * kLog2e : -INFINITY;
            cm = fmaxf(cm, v[j]);
          }
          if (cm > m2) {
            if (m2 > -INFINITY) s *= ex2_approx(m2 - cm);
            m2 = cm;
          }
          if (m2 > -INFINITY) {
#pragma unroll
            for (int j = 0; j < 32; ++j) s += ex2_approx(v[j] - m2);
          }
        }
        if (row_ok) p.part[(int64_t)c.nt * p.part_ld + grow] = make_float2(m2, s);
      } else if constexpr (KIND == TcKind::GRAD) {
        float lse2 = 0.f, gmul = 0.f;
        if (row_ok) {
          const float4 cs = p.cst[grow];
          lse2 = cs.x * kLog2e;
          gmul = cs.y;
        }
        uint16_t* grow_ptr = p.G + (int64_t)grow * p.ldG;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          float v[32];
          tmem_ld32(taddr + cc * 32, v);
          const int cb = col0 + cc * 32;
          if (!row_ok || cb >= p.V) continue;
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            pk[j] = pack_bf16x2(gmul * ex2_approx(fmaf(v[2 * j], kLog2e, -lse2)),
                                gmul * ex2_approx(fmaf(v[2 * j + 1], kLog2e, -lse2)));
          if (cb + 32 <= p.V) {
            uint4* dst = reinterpret_cast<uint4*>(grow_ptr + cb);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (cb + j < p.V)
                grow_ptr[cb + j] = (uint16_t)((j & 1) ? (pk[j >> 1] >> 16) : (pk[j >> 1] & 0xFFFFu));
          }
        }
      } else {
        // DH: fp32 partial of split c.split; DW: dW (+)= acc.
        float* out = (KIND == TcKind::DH)
                         ? p.dHp + (int64_t)c.split * p.M * p.N + (int64_t)grow * p.N
                         : p.dW + (int64_t)grow * p.N;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          float v[32];
          tmem_ld32(taddr + cc * 32, v);
          const int cb = col0 + cc * 32;
          if (!row_ok || cb >= p.N) continue;
          if (cb + 32 <= p.N) {
            float4* dst = reinterpret_cast<float4*>(out + cb);
            if (KIND == TcKind::DW && !p.first) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                float4 o = dst[j];
                o.x += v[4 * j]; o.y += v[4 * j + 1]; o.z += v[4 * j + 2]; o.w += v[4 * j + 3];
                dst[j] = o;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (cb + j < p.N)
                out[cb + j] = (KIND == TcKind::DW && !p.first) ? out[cb + j] + v[j] : v[j];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <TcKind KIND>
cudaError_t launch_kind(const TcMaps& maps, const TcLaunch& p, cudaStream_t s) {
  using L = Layout<KIND>;
  const int n_m = (p.M + BM - 1) / BM;
  const int n_n = (p.N + L::BN - 1) / L::BN;
  const int n_tiles = n_m * n_n * (KIND == TcKind::DH ? p.n_split : 1);
  if (n_tiles <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(tc_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = n_tiles < p.num_sms ? n_tiles : p.num_sms;
  tc_kernel<KIND><<<grid, kThreads, L::SMEM_BYTES, s>>>(maps.a, maps.b, p);
  return cudaGetLastError();
}

}  // namespace

int tc_bn(TcKind k) {
  switch (k) {
    case TcKind::LSE: return Cfg<TcKind::LSE>::BN;
    case TcKind::GRAD: return Cfg<TcKind::GRAD>::BN;
    case TcKind::DH: return Cfg<TcKind::DH>::BN;
    default: return Cfg<TcKind::DW>::BN;
  }
}

cudaError_t launch_tc(const TcMaps& maps, const TcLaunch& p, cudaStream_t s) {
  switch (p.kind) {
    case TcKind::LSE: return launch_kind<TcKind::LSE>(maps, p, s);
    case TcKind::GRAD: return launch_kind<TcKind::GRAD>(maps, p, s);
    case TcKind::DH: return launch_kind<TcKind::DH>(maps, p, s);
    default: return launch_kind<TcKind::DW>(maps, p, s);
  }
}

}  // namespace ckl
