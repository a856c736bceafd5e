// bf16 tensor-core contractions of the fused top-K forward-KL loss on sm_100a.
//
// One persistent, warp-specialised kernel template serves the products of the
// method ("Chunked KL loss, running Knowledge Distillation locally in less <6GB
// VRAM", README "Full Chunked KL": the logits of a chunk exist only while the
// normaliser is being accumulated, and the backward pass needs the analytic
// gradient of each chunk):
//   LSE : z = H_c W^T tile by tile; the epilogue keeps each row's (max, sum of
//         exp) over the tile's vocabulary columns, and sum_k p_k z_k over the
//         row's cached teacher ids that fall in the tile. With `store_e` it also writes
//         exp(z - r) in bf16 to the chunk's gradient buffer (r the row's reference
//         logit), so the backward pass can scale rows instead of forming z again.
//   GRAD: z formed again; the epilogue writes G = gmul * exp(z - lse) in bf16.
//   DH  : dH_c = G W, the vocabulary split in n_split ranges (fp32 partials,
//         reduced in a fixed order afterwards).
//   DW  : dW (+)= G^T H_c, contraction over the chunk's tokens; the epilogue adds
//         its fp32 tile into dW with a TMA reduce-add (the add happens in L2).
//   TKMAX, TKEMIT: the teacher top-K cache builder's two passes over the
//         teacher's logits (best logit per row and tile; candidates at least as
//         good as the row's threshold), same mainloop as LSE.
//
// Work unit: a 256 x BN output tile computed by a CTA pair (a cluster of two
// CTAs on neighbouring SMs) with tcgen05.mma.cta_group::2: each CTA stages its
// own 128 rows of A and its own BN/2 rows (K-major) or columns (MN-major) of B,
// so a stage is 32 KB per CTA and the rings hold 6-7 stages (BN = 256; a 192-wide
// dW tile with a transposed copy of H measured slower, 39 vs 34 ms per step). The pair's
// accumulator is split by rows: rows 0-127 in the even CTA's TMEM, 128-255 in the
// odd CTA's.
//
// CTA layout (192 threads, one CTA per SM, two CTAs per cluster):
//   warp 0      TMA producer (both CTAs): tiles into the CTA's own ring; the
//               copies signal the even CTA's `full` barrier, where the even
//               producer has posted the byte count of both halves.
//   warp 1      allocates 512 TMEM columns in both CTAs; in the even CTA one
//               thread issues the pair MMAs (M=256, N=256, K=16) into one of two
//               accumulators and commits each stage to the `empty` barriers of
//               both CTAs (one tcgen05.commit arriving in both).
//   warps 2..5  epilogue (both CTAs): tcgen05.ld of the CTA's 128 accumulator
//               rows (thread = row), the kind's math, plain stores or 128B-swizzled
//               staging + TMA bulk stores, then one arrival per warp on the even
//               CTA's `tempty` barrier.
// Operand layouts: H, W and G are read K-major for LSE/GRAD/DH-A; W (DH-B), G
// (DW-A) and H (DW-B) are read MN-major, so no operand is ever transposed in
// memory. Every TMA load fills the issuing CTA's own shared memory only. Every
// wait is bounded (common.cuh).
#include <atomic>

#include "common.cuh"
#include "k_tc.h"

namespace ckl {

namespace {

constexpr int BM = 128;               // rows of A per CTA (256 per pair)
constexpr int BK = 64;                // 64 bf16 = one 128-byte swizzle row
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kAccStride = 256;       // TMEM columns between the two accumulators
constexpr int kAtomBytes = 64 * 128;  // one 64 (MN) x 64 (K) MN-major box
constexpr int kStageBufBytes = 4096;  // one epilogue staging box: 32 rows x 128 bytes
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint16_t kPairMask = 0x3;
constexpr long long kPaceMaxCycles = 1LL << 22;  // bound on the measured tile time used for pacing

template <TcKind KIND>
struct Cfg;
// BN: output columns of one accumulator (each CTA stages BN/2 rows or columns of B).
// NACC: accumulators per tile. DH runs two side by side (a 256 x 512 tile): every A
// stage (G) feeds two MMAs, so a stage moves 48 KB per CTA for twice the work of a
// 32 KB single-accumulator stage, and a vocabulary split has half as many tiles
// (48 at the 32K workload, so the three splits' 144 tiles run as two waves on 74
// pairs and far fewer tiles re-stream a split's G and W from DRAM). The two
// accumulators fill all 512 TMEM columns, so that kind is single-buffered: its
// tiles run ~1000 K-blocks, against an epilogue of a few microseconds.
template <> struct Cfg<TcKind::LSE>  { static constexpr int BN = 256, NACC = 1; static constexpr bool A_MN = false, B_MN = false; static constexpr int STAGES = 6; static constexpr bool STAGED = true; };
template <> struct Cfg<TcKind::GRAD> { static constexpr int BN = 256, NACC = 1; static constexpr bool A_MN = false, B_MN = false; static constexpr int STAGES = 6; static constexpr bool STAGED = true; };
template <> struct Cfg<TcKind::DH>   { static constexpr int BN = 256, NACC = 2; static constexpr bool A_MN = false, B_MN = true;  static constexpr int STAGES = 4; static constexpr bool STAGED = false; };
template <> struct Cfg<TcKind::DW>   { static constexpr int BN = 256, NACC = 1; static constexpr bool A_MN = true,  B_MN = true;  static constexpr int STAGES = 6; static constexpr bool STAGED = true; };
template <> struct Cfg<TcKind::TKMAX>  { static constexpr int BN = 256, NACC = 1; static constexpr bool A_MN = false, B_MN = false; static constexpr int STAGES = 7; static constexpr bool STAGED = false; };
template <> struct Cfg<TcKind::TKEMIT> { static constexpr int BN = 256, NACC = 1; static constexpr bool A_MN = false, B_MN = false; static constexpr int STAGES = 7; static constexpr bool STAGED = false; };

// The bf16 gradient buffer is blocked: 64 x 64 element blocks (64 vocabulary ids
// fastest, then 64 tokens; 8 KB contiguous), seen by TMA as the 4-D tensor
// (64, 64, vocabulary blocks, token blocks). DH and DW read it as their A
// operand (DH: K-major, 128 token rows = two token blocks per box; DW: MN-major,
// two neighbouring vocabulary blocks per box, one per 64-wide atom); LSE and GRAD
// write it from their epilogues.
template <TcKind KIND>
constexpr bool kAisG = KIND == TcKind::DH || KIND == TcKind::DW;
template <TcKind KIND>
constexpr bool kCisG = KIND == TcKind::LSE || KIND == TcKind::GRAD;

template <TcKind KIND>
struct Layout {
  static constexpr int BN = Cfg<KIND>::BN;
  static constexpr int BNH = BN / 2;
  static constexpr int STAGES = Cfg<KIND>::STAGES;
  static constexpr int NACC = Cfg<KIND>::NACC;
  static constexpr int TW = BN * NACC;                  // output columns of a tile
  static constexpr int NBUF = NACC == 1 ? 2 : 1;        // accumulator buffers in TMEM
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_HALF_BYTES = BNH * BK * 2;     // one accumulator's B, this CTA's half
  static constexpr int B_BYTES = NACC * B_HALF_BYTES;
  static_assert(!Cfg<KIND>::B_MN || BNH % 64 == 0, "MN-major B is staged in 64-column atoms");
  static_assert(NACC * BN <= kTmemCols && (NBUF == 1 || NACC * BN <= kAccStride),
                "accumulators fit in TMEM");
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  // two staging boxes per epilogue warp
  static constexpr int EPI_BYTES = Cfg<KIND>::STAGED ? 4 * 2 * kStageBufBytes : 0;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + RING_BYTES + EPI_BYTES + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

struct TileCoord {
  int mt, nt, kb0, kb1, split;
};

__device__ __forceinline__ TileCoord tile_coord(const TcLaunch& p, int n_m, int n_n, int kps,
                                                int tile) {
  TileCoord c;
  c.split = 0;
  if (p.kind == TcKind::DW) {  // neighbouring pairs share the A (gradient) tile
    c.nt = tile % n_n;
    c.mt = tile / n_n;
  } else {  // neighbouring pairs share the B tile (W rows / columns)
    c.mt = tile % n_m;
    const int r = tile / n_m;
    c.nt = r % n_n;
    c.split = r / n_n;
  }
  c.kb0 = c.split * kps;
  c.kb1 = min(p.n_kb, c.kb0 + kps);
  return c;
}

// Write one thread's 128-byte row (8 x 16 bytes) into a 32-row staging box laid
// out as the 128-byte TMA swizzle expects: 16-byte chunk c of row r sits at
// position c ^ (r % 8).
__device__ __forceinline__ void stage_row(unsigned char* box, int r, const uint4 (&chunks)[8]) {
  uint4* rowp = reinterpret_cast<uint4*>(box + r * 128);
#pragma unroll
  for (int c = 0; c < 8; ++c) rowp[c ^ (r & 7)] = chunks[c];
}

// v[i] for a runtime index 0 <= i < 32, by selects (the array stays in registers).
__device__ __forceinline__ float pick32(const float (&v)[32], int i) {
  float r = v[0];
#pragma unroll
  for (int t = 1; t < 32; ++t) r = (i == t) ? v[t] : r;
  return r;
}

// Pack 32 + 32 fp32 values as 64 bf16 (one staged row of a 64-column box).
__device__ __forceinline__ void pack_row_bf16(const float (&a)[32], const float (&b)[32],
                                              uint4 (&out)[8]) {
#pragma unroll
  for (int c = 0; c < 4; ++c)
    out[c] = make_uint4(pack_bf16x2(a[8 * c], a[8 * c + 1]), pack_bf16x2(a[8 * c + 2], a[8 * c + 3]),
                        pack_bf16x2(a[8 * c + 4], a[8 * c + 5]),
                        pack_bf16x2(a[8 * c + 6], a[8 * c + 7]));
#pragma unroll
  for (int c = 0; c < 4; ++c)
    out[4 + c] = make_uint4(pack_bf16x2(b[8 * c], b[8 * c + 1]),
                            pack_bf16x2(b[8 * c + 2], b[8 * c + 3]),
                            pack_bf16x2(b[8 * c + 4], b[8 * c + 5]),
                            pack_bf16x2(b[8 * c + 6], b[8 * c + 7]));
}

template <TcKind KIND>
__global__ void __launch_bounds__(kThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmC, const TcLaunch p) {
  using L = Layout<KIND>;
  constexpr int STAGES = L::STAGES;
  constexpr int BN = L::BN, BNH = L::BNH, TW = L::TW, NACC = L::NACC, NBUF = L::NBUF;
  constexpr bool A_MN = Cfg<KIND>::A_MN, B_MN = Cfg<KIND>::B_MN;

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* epi_smem = smem + L::RING_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::RING_BYTES + L::EPI_BYTES);
  uint64_t* full = bars;                 // [STAGES] used in the even CTA
  uint64_t* empty = bars + STAGES;       // [STAGES] both CTAs
  uint64_t* tfull = bars + 2 * STAGES;   // [2] both CTAs
  uint64_t* tempty = tfull + 2;          // [2] used in the even CTA
  uint64_t* done = tempty + 2;           // [1] even CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: leader (issues MMAs), 1: peer
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int n_m = (p.M + 2 * BM - 1) / (2 * BM);
  const int n_n = (p.N + TW - 1) / TW;
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
      mbar_init(&tempty[b], 2 * 4);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (Cfg<KIND>::STAGED) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Every CTA of this persistent grid is resident: a kernel launched behind this one
  // as a dependent may take what room is left on the SMs from here on.
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_phase = 0;  // per-stage bits: loaded at least once / last parity
      bool ok = true;
      for (int tile = pair; ok && tile < n_tiles; tile += n_pairs) {
        const TileCoord c = tile_coord(p, n_m, n_n, kps, tile);
        const int a_row0 = c.mt * 2 * BM + (int)rank * BM;  // this CTA's rows of A
        const int b_row0 = c.nt * TW + (int)rank * BNH;     // this CTA's rows/columns of B
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          unsigned char* sA = smem + stage * L::STAGE_BYTES;
          unsigned char* sB = sA + L::A_BYTES;
          const uint32_t fbar = cluster_map(&full[stage], 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * L::STAGE_BYTES);
          if constexpr (kAisG<KIND> && !A_MN) {
            // 128 token rows of one 64-wide vocabulary block: two token blocks
            tma_load_4d_pair(sA, &tmA, fbar, 0, 0, kb, a_row0 >> 6);
          } else if constexpr (kAisG<KIND>) {
            // MN-major: the CTA's two 64-wide atoms are two neighbouring (contiguous)
            // blocks of one token block; one box, atom 1 landing kAtomBytes after atom 0
            tma_load_4d_pair(sA, &tmA, fbar, 0, 0, a_row0 >> 6, kb);
          } else if (!A_MN) {
            tma_load_2d_pair(sA, &tmA, fbar, kb * BK, a_row0);
          } else {
#pragma unroll
            for (int a = 0; a < BM / 64; ++a)
              tma_load_2d_pair(sA + a * kAtomBytes, &tmA, fbar, a_row0 + a * 64, kb * BK);
          }
#pragma unroll
          for (int acc = 0; acc < NACC; ++acc) {  // accumulator acc: tile columns acc * BN ...
            unsigned char* sBa = sB + acc * L::B_HALF_BYTES;
            if (!B_MN) {
              tma_load_2d_pair(sBa, &tmB, fbar, kb * BK, b_row0 + acc * BN);
            } else {
#pragma unroll
              for (int a = 0; a < BNH / 64; ++a)
                tma_load_2d_pair(sBa + a * kAtomBytes, &tmB, fbar, b_row0 + acc * BN + a * 64,
                                 kb * BK);
            }
          }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Wait until the pair's MMAs have consumed every stage this thread filled
      // (so no copy is in flight when the CTA exits).
      for (int s = 0; s < STAGES; ++s) {
        if (!((issued >> s) & 1u)) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(&empty[s], (issued_phase >> s) & 1u)) {
          if (clock64() - t0 > kWaitCycles) { atomicOr(p.status, (unsigned)ST_TIMEOUT); break; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(2 * BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < n_tiles; tile += n_pairs, ++it) {
        const TileCoord c = tile_coord(p, n_m, n_n, kps, tile);
        const int buf = NBUF == 2 ? (it & 1) : 0;
        const uint32_t use = NBUF == 2 ? (uint32_t)(it >> 1) : (uint32_t)it;
        // the second accumulator of a tile whose columns all lie past N has nothing to do
        const int n_acc = (NACC == 2 && c.nt * TW + BN >= p.N) ? 1 : NACC;
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
#pragma unroll
            for (int acc = 0; acc < NACC; ++acc) {
              if (acc >= n_acc) break;
              const uint32_t ba = b0 + acc * L::B_HALF_BYTES;
              const uint64_t bd = B_MN ? umma_desc_sw128(ba + kk * 2048, kAtomBytes, 1024)
                                       : umma_desc_sw128(ba + kk * 32, 16, 1024);
              umma_bf16_pair(d_tmem + acc * BN, ad, bd, idesc, (kb > c.kb0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit_pair_mc(&empty[stage], kPairMask);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair_mc(&tfull[buf], kPairMask);
      }
      // Every MMA issued above has completed once `done` flips.
      umma_commit_pair(done);
      const long long t0 = clock64();
      while (!mbar_try_wait(done, 0)) {
        if (clock64() - t0 > kWaitCycles) { atomicOr(p.status, (unsigned)ST_TIMEOUT); break; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;   // accumulator row owned by this thread (within the CTA)
    unsigned char* stg = epi_smem + q * 2 * kStageBufBytes;  // this warp's two staging boxes
    int nstage = 0;                  // staging boxes this warp has filled so far
    // Fill staging box (nstage & 1) from this thread's row and hand it to TMA.
    // Rows past the tensor are not stored, except in the gradient buffer: its last
    // 64-token block is read whole by DW (rows past M against zero-filled H rows),
    // so those rows must hold finite values, not what the workspace held before.
    const int row_lim = kCisG<KIND> ? ((p.M + 63) & ~63) : p.M;
    auto stage_and_issue = [&](const uint4 (&chunks)[8], int c0, int c1, bool reduce) {
      if (c1 >= row_lim) return;  // every row of this warp's box is past the limit (warp-uniform)
      unsigned char* box = stg + (nstage & 1) * kStageBufBytes;
      if (lane == 0) bulk_wait_read<1>();  // the box's previous store has read it
      __syncwarp();
      stage_row(box, lane, chunks);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kCisG<KIND>) tma_store_4d(&tmC, box, 0, c1 & 63, c0 >> 6, c1 >> 6);
        else if (reduce) tma_reduce_add_2d(&tmC, box, c0, c1);
        else tma_store_2d(&tmC, box, c0, c1);
        bulk_commit();
      }
      ++nstage;
    };

    if constexpr (KIND == TcKind::DH) {
      // The scaled hidden states the dW contraction reads, written while these warps
      // would otherwise wait for their first accumulator (~a millisecond away).
      if (p.Hs) {
        const int64_t n8 = (int64_t)p.M * p.N / 8;
        const int64_t step = (int64_t)gridDim.x * 128;
        for (int64_t e = (int64_t)blockIdx.x * 128 + (threadIdx.x - 64); e < n8; e += step)
          scale_h8(p.Hc, p.Hs, e * 8, row_factor(p.cst, e * 8 / p.N));
      }
    }
    int it = 0;
    long long t_prev = 0;  // when the previous tile's accumulator became ready (SM cycles)
    for (int tile = pair; tile < n_tiles; tile += n_pairs, ++it) {
      const TileCoord c = tile_coord(p, n_m, n_n, kps, tile);
      const int buf = NBUF == 2 ? (it & 1) : 0;
      const uint32_t use = NBUF == 2 ? (uint32_t)(it >> 1) : (uint32_t)it;
      if (!mbar_wait(&tfull[buf], use & 1u, abort_flag, p.status)) break;
      tc_fence_after();
      // The MMA time of one tile, measured as the distance between consecutive
      // accumulators becoming ready (0 for the first tile), bounded.
      const long long t_now = clock64();
      const long long t_tile = t_prev > 0 ? min(t_now - t_prev, (long long)kPaceMaxCycles) : 0;
      t_prev = t_now;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kAccStride);
      const int crow0 = c.mt * 2 * BM + (int)rank * BM;  // first output row of this CTA
      const int grow = crow0 + row;  // output row (token for LSE/GRAD/DH, vocab id for DW)
      const bool row_ok = grow < p.M;
      const int col0 = c.nt * TW;
      const int row0 = crow0 + q * 32;  // first row of this warp's staging boxes

      if constexpr (KIND == TcKind::LSE) {
        // (max, sum exp2) over the tile's valid columns, in log2 units; on the same
        // pass, sum p_k z_k over the row's cached ids that fall in this tile (the
        // ids are sorted, so a cursor advances with the columns).
        const int32_t* srow = p.sid + (int64_t)grow * p.K;
        const float* prow = p.sp + (int64_t)grow * p.K;
        int j = p.K;
        if (row_ok) {
          int lo = 0, hi = p.K;  // first sorted id >= col0
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(srow + mid) < col0) lo = mid + 1; else hi = mid;
          }
          j = lo;
        }
        int nid = j < p.K ? __ldg(srow + j) : INT_MAX;
        float cross = 0.f;
        float m2 = -INFINITY;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          float v[32];
          tmem_ld32(taddr + cc * 32, v);
          const int cb = col0 + cc * 32;
          while (nid < cb + 32) {
            if (nid < p.V) cross += __ldg(prow + j) * pick32(v, nid - cb);
            ++j;
            nid = j < p.K ? __ldg(srow + j) : INT_MAX;
          }
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if (cb + jj < p.V) m2 = fmaxf(m2, v[jj] * kLog2e);
        }
        if (row_ok) p.xpart[(int64_t)c.nt * p.part_ld + grow] = cross;
        float s = 0.f;
        if (!p.store_e) {
#pragma unroll 1
          for (int cc = 0; cc < BN / 32; ++cc) {
            float v[32];
            tmem_ld32(taddr + cc * 32, v);
            const int cb = col0 + cc * 32;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              s += (cb + j < p.V) ? ex2_approx(fmaf(v[j], kLog2e, -m2)) : 0.f;
          }
        } else {
          // e = exp2(z log2e - m2) in (0, 1] enters the sum; the value stored (bf16, 64
          // columns at a time) is e * exp2(m2 - ref) = exp2(z log2e - ref), with ref the
          // row's reference unless this tile's maximum lies more than kRefGap above it
          const float r2 = row_ok ? p.tok[grow].w : m2;
          const float ref = m2 > r2 + kRefGap ? m2 : r2;
          const float fs = ex2_approx(m2 - ref);
#pragma unroll 1
          for (int cc = 0; cc < BN / 64; ++cc) {
            // the 64 KB a CTA stores per tile leave in four groups spread over the
            // next tile's MMA time (group cc at cc/6 of it), as in the dW epilogue
            if (cc > 0 && t_tile > 0) {
              const long long due = t_now + t_tile * cc / 6;
              while (clock64() < due) __nanosleep(128);
            }
            float a[32], b[32];
            tmem_ld32(taddr + cc * 64, a);
            tmem_ld32(taddr + cc * 64 + 32, b);
            const int cb = col0 + cc * 64;
            // same expressions and summation order (column by column) as above,
            // so lse does not depend on whether e is stored
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              a[j] = (cb + j < p.V) ? ex2_approx(fmaf(a[j], kLog2e, -m2)) : 0.f;
              s += a[j];
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              b[j] = (cb + 32 + j < p.V) ? ex2_approx(fmaf(b[j], kLog2e, -m2)) : 0.f;
              s += b[j];
            }
            if (cb < p.V) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                a[j] *= fs;
                b[j] *= fs;
              }
              uint4 ch[8];
              pack_row_bf16(a, b, ch);
              stage_and_issue(ch, cb, row0, false);
            }
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
#pragma unroll 1
        for (int cc = 0; cc < BN / 64; ++cc) {
          if (cc > 0 && t_tile > 0) {  // stores spread over the next tile, as in LSE
            const long long due = t_now + t_tile * cc / 6;
            while (clock64() < due) __nanosleep(128);
          }
          float a[32], b[32];
          tmem_ld32(taddr + cc * 64, a);
          tmem_ld32(taddr + cc * 64 + 32, b);
          const int cb = col0 + cc * 64;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            a[j] = gmul * ex2_approx(fmaf(a[j], kLog2e, -lse2));
            b[j] = gmul * ex2_approx(fmaf(b[j], kLog2e, -lse2));
          }
          if (cb < p.V) {
            uint4 ch[8];
            pack_row_bf16(a, b, ch);
            stage_and_issue(ch, cb, row0, false);
          }
        }
      } else if constexpr (KIND == TcKind::TKMAX) {
        // the row's best logit in this vocabulary tile and its smallest id
        float best = -INFINITY;
        int bid = INT_MAX;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          float v[32];
          tmem_ld32(taddr + cc * 32, v);
          const int cb = col0 + cc * 32;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (cb + j < p.V && v[j] > best) { best = v[j]; bid = cb + j; }
        }
        if (row_ok) p.part[(int64_t)c.nt * p.part_ld + grow] = make_float2(best, __int_as_float(bid));
      } else if constexpr (KIND == TcKind::TKEMIT) {
        // every (logit, id) at least as good as the row's threshold joins its candidates
        float tv = INFINITY;
        int tid = -1;
        if (row_ok) {
          const float2 th = p.theta[grow];
          tv = th.x;
          tid = __float_as_int(th.y);
        }
        int* cnt = p.cand_cnt + grow;
        float2* crow = p.cand + (int64_t)grow * p.cand_cap;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          float v[32];
          tmem_ld32(taddr + cc * 32, v);
          const int cb = col0 + cc * 32;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = cb + j;
            if (col < p.V && (v[j] > tv || (v[j] == tv && col <= tid))) {
              const int slot = atomicAdd(cnt, 1);
              if (slot < p.cand_cap) crow[slot] = make_float2(v[j], __int_as_float(col));
            }
          }
        }
      } else if constexpr (KIND == TcKind::DH) {
        // fp32 partial of split c.split, plain vector stores
        float* out = p.dHp + (int64_t)c.split * p.M * p.N + (int64_t)grow * p.N;
#pragma unroll 1
        for (int cc = 0; cc < TW / 32; ++cc) {
          const int cb = col0 + cc * 32;
          if (cb >= p.N && (cb - col0) % BN == 0) break;  // an accumulator past N: not computed
          float v[32];
          tmem_ld32(taddr + cc * 32, v);
          if (!row_ok || cb >= p.N) continue;
          if (cb + 32 <= p.N) {
            float4* dst = reinterpret_cast<float4*>(out + cb);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (cb + j < p.N) out[cb + j] = v[j];
          }
        }
      } else {
        // DW: stage 32 fp32 columns per box and add them into dW in L2
        // (store instead of add for the first chunk). Every pair finishes its tiles
        // at about the same moment and each add misses L2 (dW is 2.3 GB), so
        // issuing a whole tile's 128 KB per CTA at once floods L2 and DRAM just as
        // the next tile's operand loads go out, and the MMA waits on them. Box group
        // cc therefore leaves cc/10 of a tile's MMA time after the accumulator is
        // ready (the last at 0.7 of it, well before this buffer is needed again).
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          if (cc > 0 && t_tile > 0) {
            const long long due = t_now + t_tile * cc / 10;
            while (clock64() < due) __nanosleep(128);
          }
          float v[32];
          tmem_ld32(taddr + cc * 32, v);
          const int cb = col0 + cc * 32;
          if (cb >= p.N) continue;
          uint4 ch[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            ch[j] = make_uint4(__float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                               __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
          stage_and_issue(ch, cb, row0, !p.first);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_map(&tempty[buf], 0));
    }
    if (Cfg<KIND>::STAGED && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <TcKind KIND>
cudaError_t launch_kind(const TcMaps& maps, const TcLaunch& p, cudaStream_t s) {
  using L = Layout<KIND>;
  const int n_m = (p.M + 2 * BM - 1) / (2 * BM);
  const int n_n = (p.N + L::TW - 1) / L::TW;
  const int n_tiles = n_m * n_n * (KIND == TcKind::DH ? p.n_split : 1);
  if (n_tiles <= 0) return cudaSuccess;
  // The shared-memory attribute is per device: set it once per device (bit per ordinal),
  // so a call made during stream capture issues no attribute change.
  static std::atomic<uint64_t> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (!bit || !(attr_set.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(tc_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // As many pairs as can be resident at once (one CTA per SM), at most one per tile.
  // Cached per kind; concurrent first calls compute the same value.
  static std::atomic<int> cached_pairs{0};
  int max_pairs = cached_pairs.load(std::memory_order_relaxed);
  if (max_pairs == 0) {
    cfg.gridDim = dim3(2 * p.num_sms, 1, 1);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, tc_kernel<KIND>, &cfg) != cudaSuccess ||
        clusters < 1)
      clusters = p.num_sms / 2;
    max_pairs = clusters;
    cached_pairs.store(max_pairs, std::memory_order_relaxed);
  }
  const int pairs = n_tiles < max_pairs ? n_tiles : max_pairs;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  return cudaLaunchKernelEx(&cfg, tc_kernel<KIND>, maps.a, maps.b, maps.c, p);
}

}  // namespace

int tc_bn(TcKind k) {
  switch (k) {
    case TcKind::LSE: return Layout<TcKind::LSE>::TW;
    case TcKind::GRAD: return Layout<TcKind::GRAD>::TW;
    case TcKind::DH: return Layout<TcKind::DH>::TW;
    case TcKind::TKMAX: return Layout<TcKind::TKMAX>::TW;
    case TcKind::TKEMIT: return Layout<TcKind::TKEMIT>::TW;
    default: return Layout<TcKind::DW>::TW;
  }
}

cudaError_t launch_tc(const TcMaps& maps, const TcLaunch& p, cudaStream_t s) {
  switch (p.kind) {
    case TcKind::LSE: return launch_kind<TcKind::LSE>(maps, p, s);
    case TcKind::GRAD: return launch_kind<TcKind::GRAD>(maps, p, s);
    case TcKind::DH: return launch_kind<TcKind::DH>(maps, p, s);
    case TcKind::TKMAX: return launch_kind<TcKind::TKMAX>(maps, p, s);
    case TcKind::TKEMIT: return launch_kind<TcKind::TKEMIT>(maps, p, s);
    default: return launch_kind<TcKind::DW>(maps, p, s);
  }
}

}  // namespace ckl
