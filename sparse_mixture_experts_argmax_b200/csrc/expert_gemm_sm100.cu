// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM),
// bf16 inputs with fp32 accumulation.
//
// Each expert is an FFN, E_i(x) = W_2,i relu(W_1,i x + b_1,i) + b_2,i, and a
// kept token's layer output is y_t = g_t E_{e_t}(x_t) (Switch Transformer
// reading note, sections "Expert FFN Layer" and "Router").  The expert
// computation is a batched matrix multiplication over the tokens each expert
// received (paper-graph summary of arXiv 2101.03961, "The routing mechanics in
// detail": expert computation).
//
//   GEMM1 (which = 0): hbuf[r, :]  = relu(W1[e] xbuf[r, :] + b1[e])        (bf16)
//   GEMM2 (which = 1): out[tok, :] = g_tok * (W2[e] hbuf[r, :] + b2[e])     (bf16)
//                      with tok = slot_token[r]: the scatter back to token order
//                      (the combine) happens in this epilogue.
//
// Formulation ("swap AB"): the weight matrix is the UMMA A operand (M = 128
// output features per tile, K-major), the packed token rows of one expert are
// the B operand (N = up to 256 tokens, K-major), so every weight byte is
// streamed from HBM once per token tile no matter how few tokens an expert has.
// D[feature, token] accumulates in TMEM.
//
// Persistent kernel, one CTA per SM, 384 threads:
//   warp 0      TMA producer (one thread): A and B k-blocks of 64 elements into a
//               ring of shared-memory stages (128-byte swizzle)
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma (K = 16) per stage
//   warp 2      TMEM allocator (512 columns: four 128-column accumulators for
//               token tiles of up to 128 rows, else two of 256)
//   warp 3      tile scheduler (one thread): claims, decodes and publishes tiles
//   warps 4..11 epilogue, two warps per TMEM lane quarter taking alternate
//               32-column chunks: tcgen05.ld, bias / ReLU / gate in fp32, bf16
//               pack, transpose through shared memory, 16-byte stores
// Tiles (expert, 128-feature block, token block) are numbered expert-major and
// handed out in order by a device counter, every tile (a CTA's first included)
// claimed by a CTA that is already running; the token-block count of each
// expert comes from the device tile prefix written by the dispatch scan.  The
// scheduler keeps the claim, the decode (dependent loads of the prefix) and the
// GEMM2 readiness wait off the producer's path.  Within an expert the tiles go
// token block by token block when its weights fit in L2 (the first blocks'
// GEMM2 can start while GEMM1 of the last ones runs).  Layers with a long GEMM2
// reduction cut their GEMM2 tiles over K (the kSplit instantiation): each
// sub-tile stores an fp32 partial and ffn_split_reduce_kernel, launched after,
// adds them in k order and stores the rows.  Every wait is bounded; a stuck
// pipeline sets the device error word and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace swl {
namespace {

constexpr int kEpiWarps = 8;          // two per TMEM lane quarter, alternating column chunks
constexpr int kThreads = 128 + 32 * kEpiWarps;
constexpr int kBM = 128;              // UMMA M: output features per tile
constexpr int kBK = 64;               // K elements per stage (one 128-byte swizzle row)
constexpr int kUmmaK = 16;            // K per tcgen05.mma (bf16)
constexpr int kMaxStages = 12;
constexpr int kMaxAcc = 4;            // TMEM accumulator buffers (512 / acc_cols)
constexpr int kTmemCols = 512;
constexpr uint32_t kABytes = kBM * kBK * 2;   // 16 KiB
constexpr int kEpiStageBytes = kEpiWarps * 32 * 32 * 2;   // per-warp 32x32 bf16 transpose tiles
constexpr int kMaxPending = 2;        // GEMM1 tiles an epilogue warp publishes per fence

// One GEMM of the expert FFN.
struct PhaseArgs {
  const __nv_bfloat16* bias;   // [N, M]
  __nv_bfloat16* out;          // GEMM1: hbuf [T, M] (packed rows); GEMM2: out [T, M]
  int M;          // output features per expert
  int a_rows;     // rows of the A operand per expert: M, or 2 M for GEGLU (gate rows,
                  // then value rows); also the bias stride per expert
  int m_tiles;    // ceil(M / 128)
  int k_blocks;   // ceil(K / 64)
  int mode;       // 0: bias + ReLU, packed rows; 1: bias, gate, scatter to token rows;
                  // 2: bias only, packed rows (expert-parallel: the gate is applied
                  //    on the rank that holds the token)
};

struct FfnArgs {
  const int* tile_prefix;      // [N+1] token tiles before expert e
  const int* exp_rows;         // [N]
  const int* exp_base;         // [N]
  const float* gate;           // [T]
  const int* slot_token;       // [T]
  int* ready;                  // [token tiles] GEMM1 epilogue warps finished (zeroed by the scan)
  unsigned int* next_tile;     // work counter (zeroed by the scan)
  int* err;
  unsigned long long wait_ns;  // bound of every wait
  int stall_test;  // 1: token tile 0's GEMM2 readiness target is one warp too high (the
                   // wait runs out: a test of the failure path)
  int num_experts;
  int T_rows;         // rows of the packed buffers and of out (range checks)
  int cache_prefix;   // 1: the scheduler keeps the tile prefix in shared memory
  int bn;         // token rows per tile (multiple of 16, <= 256)
  int stages;
  int num_acc;    // TMEM accumulators: 4 of 128 columns when bn <= 128, else 2 of 256
                  // (GEGLU: 512 / the next power of two >= max(128, 2 bn))
  // GEMM2 split over K (split > 1): the GEMM2 tiles of the experts the
  // dispatch scan marks (split_base >= 0) are cut into `split` sub-tiles of
  // consecutive k-blocks; each sub-tile stores its fp32 partial tile, and
  // ffn_split_reduce_kernel adds the partials in k order and stores the result
  // (bias, gate, scatter) once the FFN has finished.
  int split;
  const int* tile_prefix2;     // [N+1] GEMM2 tile prefix counting split sub-tiles
  const int* split_base;       // [N] first split group of expert e, -1: not split
  float* part;                 // [groups][split][bn][128] fp32 partial tiles
  // [kSplitMaxGroups][kSplitFactor]: per token tile of a split expert (its
  // token tiles come first, so g < kSplitMaxGroups) and K chunk of GEMM2, the
  // GEMM1 epilogue warps of the tiles whose features fall in that chunk that
  // have stored their rows.  A split sub-tile waits for its own chunk only, and
  // a split expert's tiles go chunk by chunk (GEMM1: its 128-feature tiles in
  // `split` runs of consecutive tiles; GEMM2: k-chunk slowest), so the first
  // chunks' GEMM2 work is ready while the last GEMM1 tiles run.
  int* split_ready;
  // 1: within an expert, tiles go token tile by token tile (all m-tiles of
  // token tile 0 first), so that GEMM2 of the first token tiles can start
  // while GEMM1 of the last ones runs; 0: m-tile by m-tile (token tiles
  // fastest: the CTAs running together share a weight tile)
  int tok_major;
  int glu;        // 1: GEMM1 is GEGLU: each tile multiplies the gate and the value
                  // rows of W1 for the same 128 features into the two halves of
                  // its accumulator, and the epilogue stores GELU(gate) * value
  PhaseArgs ph[2];
};

struct TileCoord {
  int phase, e, mt, nt, g;   // g: global token-tile index P[e] + nt
  int ks, nsplit;            // GEMM2 split: sub-tile ks of nsplit (1: not split)
};

// A decoded work item, published by the scheduler warp in shared memory.
struct TileSlot {
  int t;          // tile id; -1: no more work
  int phase, e, mt, nt, g;
  int rows;       // valid token rows of the tile
  int row0;       // first packed row of the tile
  int kb0, kb1;   // k-blocks [kb0, kb1) of this (sub-)tile
  int ks, nsplit; // GEMM2 split: sub-tile ks of nsplit
  int grp;        // split group (partials and counters), -1: not split
  int* rdy0;      // GEMM1: the readiness counters its epilogue warps increment
  int* rdy1;      //        (rdy1: a second K chunk of a split expert, or null)
};

constexpr int kTileRing = 8;    // decoded tiles handed to the producer, MMA and epilogue

// Work item t: GEMM1 tiles [0, total0) then GEMM2 tiles.  Within a phase, the
// tiles of expert e occupy [P[e]*m_tiles, P[e+1]*m_tiles) (P = tile prefix) with
// token blocks fastest, so CTAs working at the same time share weights.
// P is the tile prefix, in shared memory when it fits there, else global.
// With a GEMM2 split, GEMM2 tiles follow the split prefix P2 instead (an
// expert's tiles there are its token tiles times its split factor).
template <bool kSplit>
__device__ __forceinline__ TileCoord decode_tile(int t, const FfnArgs& a, int total0,
                                                 const int* P) {
  TileCoord c;
  c.phase = t < total0 ? 0 : 1;
  const int tile = c.phase == 0 ? t : t - total0;
  const int m_tiles = a.ph[c.phase].m_tiles;
  const int q = tile / m_tiles;
  const int* Q = (kSplit && c.phase == 1) ? a.tile_prefix2 : P;
  int lo = 0, hi = a.num_experts;     // last e with Q[e] <= q  (Q[N] > q)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (Q[mid] <= q) lo = mid; else hi = mid;
  }
  const int p0 = P[lo];
  const int nts = P[lo + 1] - p0;
  const int q0 = Q[lo];
  const int nts2 = Q[lo + 1] - q0;     // token tiles times the split factor
  const int local = tile - q0 * m_tiles;
  c.e = lo;
  c.nsplit = nts2 / nts;
  if (kSplit && c.phase == 1 && c.nsplit > 1) {
    // split GEMM2 tiles: K chunk slowest, then the usual order within a chunk
    const int per_ks = nts * m_tiles;
    c.ks = local / per_ks;
    const int r = local - c.ks * per_ks;
    if (a.tok_major) {
      c.nt = r / m_tiles;
      c.mt = r - c.nt * m_tiles;
    } else {
      c.mt = r / nts;
      c.nt = r - c.mt * nts;
    }
  } else if (kSplit && c.phase == 0 && __ldg(a.split_base + lo) >= 0) {
    // GEMM1 tiles of a split expert: runs of mg consecutive feature tiles (one
    // run per K chunk of GEMM2), the expert's token tiles within a run
    const int mg = (m_tiles + a.split - 1) / a.split;
    const int run = local / (nts * mg);
    const int r = local - run * nts * mg;
    const int mg_r = min(mg, m_tiles - run * mg);
    c.nt = r / mg_r;
    c.mt = run * mg + (r - c.nt * mg_r);
    c.ks = 0;
  } else if (a.tok_major) {
    const int per_nt = m_tiles * c.nsplit;   // the tiles of one token tile
    c.nt = local / per_nt;
    const int r = local - c.nt * per_nt;
    c.mt = r / c.nsplit;
    c.ks = r - c.mt * c.nsplit;
  } else {
    c.mt = local / nts2;
    const int r = local - c.mt * nts2;
    c.nt = r / c.nsplit;
    c.ks = r - c.nt * c.nsplit;
  }
  c.g = p0 + c.nt;
  return c;
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Both GEMMs of the expert FFN in one persistent launch.  GEMM2 tiles of token
// tile g wait until every GEMM1 epilogue warp of g has stored its rows of hbuf.
// kGlu: GEMM1 is GEGLU (args.glu); kSplit: GEMM2 split over K (args.split > 1).
// Each is a separate instantiation so the plain kernel keeps its register budget.
template <bool kGlu, bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
expert_ffn_sm100_kernel(const __grid_constant__ CUtensorMap tmA0,
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ CUtensorMap tmB1, const FfnArgs args) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = args.stages;
  const uint32_t b_bytes = static_cast<uint32_t>(args.bn) * kBK * 2;
  constexpr uint32_t a_stage = kGlu ? 2 * kABytes : kABytes;   // A bytes per stage
  uint8_t* smem_a = smem;
  uint8_t* smem_b = smem_a + stages * a_stage;
  __nv_bfloat16* epi = reinterpret_cast<__nv_bfloat16*>(smem_b + stages * b_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(epi) + kEpiStageBytes);
  uint64_t* full_bar = bars;                      // [kMaxStages]
  uint64_t* empty_bar = bars + kMaxStages;        // [kMaxStages]
  uint64_t* tfull_bar = bars + 2 * kMaxStages;    // [kMaxAcc]
  uint64_t* tempty_bar = tfull_bar + kMaxAcc;     // [kMaxAcc]
  uint64_t* drain_bar = tempty_bar + kMaxAcc;     // [1]
  uint64_t* tile_full = drain_bar + 1;            // [kTileRing]
  uint64_t* tile_empty = tile_full + kTileRing;   // [kTileRing]
  uint64_t* take_bar = tile_empty + kTileRing;    // [1] the producer took a tile
  TileSlot* tile_ring = reinterpret_cast<TileSlot*>(take_bar + 1);   // [kTileRing]
  int* s_prefix = reinterpret_cast<int*>(tile_ring + kTileRing);      // [N+1] if cached
  uint32_t* tmem_slot =
      reinterpret_cast<uint32_t*>(s_prefix + (args.cache_prefix ? args.num_experts + 1 : 0));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(&full_bar[s], 1);
      ptx::mbar_init(&empty_bar[s], 1);
    }
    for (int i = 0; i < kMaxAcc; ++i) {
      ptx::mbar_init(&tfull_bar[i], 1);
      ptx::mbar_init(&tempty_bar[i], kEpiWarps);   // one arrive per epilogue warp
    }
    ptx::mbar_init(drain_bar, 1);
    for (int i = 0; i < kTileRing; ++i) {
      ptx::mbar_init(&tile_full[i], 1);        // the scheduler publishes a tile
      ptx::mbar_init(&tile_empty[i], kEpiWarps);   // the epilogue warps retire it
    }
    ptx::mbar_init(take_bar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tmap(&tmA0);
    ptx::prefetch_tmap(&tmB0);
    ptx::prefetch_tmap(&tmA1);
    ptx::prefetch_tmap(&tmB1);
  }
  if (warp == 2) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int acc_cols = kTmemCols / args.num_acc;
  pdl_wait();   // tile prefix, packed rows, gate and counters come from earlier kernels
  const int ntiles = args.tile_prefix[args.num_experts];
  const int total0 = ntiles * args.ph[0].m_tiles;
  const int ntiles2 = kSplit ? args.tile_prefix2[args.num_experts] : ntiles;
  const int total = total0 + ntiles2 * args.ph[1].m_tiles;

  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(args.err, kDevPipelineTimeout);
  };

  if (warp == 3) {
    // ------------------------------------------------------------ tile scheduler
    // Claims the next tile only once the producer has taken the previous one (so
    // a CTA holds at most one claimed tile it has not started), decodes it, waits
    // for its GEMM1 rows when it is a GEMM2 tile, and publishes it in the ring.
    // Every tile comes from the counter, so only a running CTA owns a tile: when
    // a GEMM2 tile is claimed, every GEMM1 tile (lower numbers) has already been
    // claimed by a running CTA, whose pipeline finishes it without waiting on
    // anything but its own stages (its epilogue publishes before it blocks), so
    // the readiness wait below ends even when other kernels hold some SMs.
    const int* P = args.tile_prefix;
    if (args.cache_prefix) {
      for (int e = lane; e <= args.num_experts; e += 32) s_prefix[e] = args.tile_prefix[e];
      __syncwarp();
      P = s_prefix;
    }
    if (lane == 0) {
      for (int i = 0;; ++i) {
        const int slot = i % kTileRing;
        if (i > 0 && !ptx::mbar_wait(take_bar, static_cast<uint32_t>(i - 1) & 1u, abort_flag, args.wait_ns)) {
          fail();
          break;
        }
        if (!ptx::mbar_wait(&tile_empty[slot], ((i / kTileRing) & 1) ^ 1u, abort_flag, args.wait_ns)) {
          fail();
          break;
        }
        const unsigned int claimed = atomicAdd(args.next_tile, 1u);
        TileSlot ts;
        ts.t = claimed < static_cast<unsigned int>(total) ? static_cast<int>(claimed) : -1;
        ts.phase = ts.e = ts.mt = ts.nt = ts.g = ts.rows = ts.row0 = 0;
        ts.kb0 = ts.kb1 = ts.ks = 0;
        ts.nsplit = 1;
        ts.grp = -1;
        ts.rdy0 = ts.rdy1 = nullptr;
        if (ts.t >= 0) {
          const TileCoord c = decode_tile<kSplit>(ts.t, args, total0, P);
          ts.phase = c.phase;
          ts.e = c.e;
          ts.mt = c.mt;
          ts.nt = c.nt;
          ts.g = c.g;
          ts.rows = min(args.bn, __ldg(args.exp_rows + c.e) - c.nt * args.bn);
          ts.row0 = __ldg(args.exp_base + c.e) + c.nt * args.bn;
          const int kbs = args.ph[c.phase].k_blocks;
          ts.ks = c.ks;
          ts.nsplit = c.nsplit;
          if (kSplit && c.nsplit > 1) {
            const int per = (kbs + c.nsplit - 1) / c.nsplit;
            ts.kb0 = c.ks * per;
            ts.kb1 = min(kbs, ts.kb0 + per);
            const int nts = P[c.e + 1] - P[c.e];
            ts.grp = __ldg(args.split_base + c.e) + c.mt * nts + c.nt;
          } else {
            ts.kb0 = 0;
            ts.kb1 = kbs;
          }
          // K chunk of GEMM2 (features of hbuf) for the split experts' counters
          const int kchunk = kSplit ? (args.ph[1].k_blocks + args.split - 1) / args.split * kBK : kBK;
          if (c.phase == 0) {
            ts.rdy0 = args.ready + c.g;
            if (kSplit && __ldg(args.split_base + c.e) >= 0) {
              // the chunks this tile's features [f0, f1] fall in
              const int f0 = c.mt * kBM, f1 = min(args.ph[0].M, f0 + kBM) - 1;
              const int c0 = f0 / kchunk, c1 = min(args.split - 1, f1 / kchunk);
              if (!checked_index(c.g >= 0 && c.g < kSplitMaxGroups && c0 <= c1, args.err)) {
                fail();
                break;
              }
              ts.rdy0 = args.split_ready + c.g * kSplitFactor + c0;
              ts.rdy1 = c1 != c0 ? args.split_ready + c.g * kSplitFactor + c1 : nullptr;
            }
          } else {
            // hbuf rows of token tile g: every GEMM1 epilogue warp of g has stored
            // them (of a split sub-tile: every warp of the GEMM1 tiles of its chunk)
            const int* rp = args.ready + c.g;
            int target = kEpiWarps * args.ph[0].m_tiles;
            if (kSplit && c.nsplit > 1) {
              const int f0 = c.ks * kchunk, f1 = min(args.ph[0].M, f0 + kchunk) - 1;
              if (!checked_index(c.g >= 0 && c.g < kSplitMaxGroups && f0 <= f1, args.err)) {
                fail();
                break;
              }
              rp = args.split_ready + c.g * kSplitFactor + c.ks;
              target = kEpiWarps * (f1 / kBM - f0 / kBM + 1);
            }
            target += args.stall_test && c.g == 0;
            bool ready = ld_acquire(rp) >= target;
            const uint64_t t0 = ptx::globaltimer_ns();
            while (!ready) {
              if (*abort_flag || ptx::globaltimer_ns() - t0 > args.wait_ns) break;
              // the counter lives in one L2 slice that many SMs may poll while
              // the epilogue warps of the GEMM1 tiles update it: poll sparingly
              __nanosleep(256);
              ready = ld_acquire(rp) >= target;
            }
            if (!ready) {
              fail();
              break;
            }
          }
        }
        tile_ring[slot] = ts;
        ptx::mbar_arrive(&tile_full[slot]);
        if (ts.t < 0) break;
      }
    }
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = ptx::l2_policy_evict_first();
      const uint64_t pol_x = ptx::l2_policy_evict_last();
      uint32_t issued = 0u;           // stages that received at least one load
      uint32_t last_par = 0u;         // parity of each stage's latest load
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int slot = i % kTileRing;
        if (!ptx::mbar_wait(&tile_full[slot], (i / kTileRing) & 1, abort_flag, args.wait_ns)) {
          fail();
          break;
        }
        const TileSlot ts = tile_ring[slot];
        if (ts.t < 0) break;
        ptx::mbar_arrive(take_bar);   // the scheduler may claim the next tile
        const PhaseArgs& P = args.ph[ts.phase];
        const CUtensorMap* tA = ts.phase == 0 ? &tmA0 : &tmA1;
        const CUtensorMap* tB = ts.phase == 0 ? &tmB0 : &tmB1;
        // GEMM2 tile: the scheduler saw the hbuf rows published (generic-proxy
        // stores of other CTAs); order them before the TMA reads below
        if (ts.phase == 1) fence_proxy_async_global();
        const int arow = ts.e * P.a_rows + ts.mt * kBM;
        const int brow = ts.row0;
        const bool two_a = kGlu && ts.phase == 0;   // gate and value rows
        if (!checked_index(ts.e >= 0 && ts.e < args.num_experts && brow >= 0 &&
                               brow + ts.rows <= args.T_rows && ts.rows > 0,
                           args.err)) {
          fail();
          break;
        }
        for (int kb = ts.kb0; kb < ts.kb1; ++kb) {
          if (!ptx::mbar_wait(&empty_bar[stage], ph ^ 1u, abort_flag, args.wait_ns)) { fail(); ok = false; break; }
          ptx::mbar_arrive_expect_tx(&full_bar[stage], (two_a ? 2 * kABytes : kABytes) + b_bytes);
          ptx::tma_load_2d(smem_a + stage * a_stage, tA, &full_bar[stage], kb * kBK, arow, pol_w);
          if (two_a)
            ptx::tma_load_2d(smem_a + stage * a_stage + kABytes, tA, &full_bar[stage], kb * kBK,
                             arow + P.M, pol_w);
          ptx::tma_load_2d(smem_b + stage * b_bytes, tB, &full_bar[stage], kb * kBK, brow, pol_x);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (ph << stage);
          if (++stage == stages) { stage = 0; ph ^= 1u; }
        }
      }
      // drain: every issued load must land before the CTA may exit
      for (int s = 0; s < stages; ++s) {
        if (issued & (1u << s)) {
          volatile int never = 0;
          if (!ptx::mbar_wait(&full_bar[s], (last_par >> s) & 1u, &never, args.wait_ns)) {
            atomicExch(args.err, kDevPipelineTimeout);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int slot = i % kTileRing;
        if (!ptx::mbar_wait(&tile_full[slot], (i / kTileRing) & 1, abort_flag, args.wait_ns)) { fail(); break; }
        const TileSlot ts = tile_ring[slot];
        if (ts.t < 0) break;
        const uint32_t n_mma = static_cast<uint32_t>((ts.rows + 15) & ~15);
        const uint32_t idesc = ptx::umma_idesc_bf16_f32(n_mma);
        if (!ptx::mbar_wait(&tempty_bar[acc], aph ^ 1u, abort_flag, args.wait_ns)) { fail(); break; }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * acc_cols);
        const bool two_a = kGlu && ts.phase == 0;   // value rows into the upper half
        const uint32_t d_val = d_tmem + static_cast<uint32_t>(acc_cols / 2);
        for (int kb = ts.kb0; kb < ts.kb1; ++kb) {
          if (!ptx::mbar_wait(&full_bar[stage], ph, abort_flag, args.wait_ns)) { fail(); ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t a_addr = ptx::smem_u32(smem_a + stage * a_stage);
          const uint32_t b_addr = ptx::smem_u32(smem_b + stage * b_bytes);
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k) {
            const uint64_t ad = ptx::umma_desc_sw128_kmajor(a_addr + k * kUmmaK * 2);
            const uint64_t bd = ptx::umma_desc_sw128_kmajor(b_addr + k * kUmmaK * 2);
            const uint32_t acc_on = (kb != ts.kb0 || k != 0) ? 1u : 0u;
            ptx::umma_bf16(d_tmem, ad, bd, idesc, acc_on);
            if (two_a) {
              const uint64_t av = ptx::umma_desc_sw128_kmajor(a_addr + kABytes + k * kUmmaK * 2);
              ptx::umma_bf16(d_val, av, bd, idesc, acc_on);
            }
          }
          ptx::umma_commit(&empty_bar[stage]);      // frees the stage when these MMAs finish
          if (++stage == stages) { stage = 0; ph ^= 1u; }
        }
        if (!ok) break;
        ptx::umma_commit(&tfull_bar[acc]);          // accumulator ready for the epilogue
        if (++acc == args.num_acc) { acc = 0; aph ^= 1u; }
      }
      // drain: all MMAs issued by this thread complete before TMEM is released
      ptx::umma_commit(drain_bar);
      volatile int never = 0;
      if (!ptx::mbar_wait(drain_bar, 0u, &never, args.wait_ns)) atomicExch(args.err, kDevPipelineTimeout);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                        // TMEM lane quarter of this warp
    const int half = (warp - 4) >> 2;              // column chunks half, half + 2, ...
    __nv_bfloat16* st = epi + (warp - 4) * 32 * 32;   // [32 tokens][32 features]
    // GEMM1 tiles whose hbuf rows this warp stored but has not yet published:
    // one fence covers up to kMaxPending of them.  The warp publishes before it
    // could block, so a GEMM2 tile never waits on a warp that is itself waiting.
    // counters of the unpublished GEMM1 tiles (warp-uniform; b: a second chunk)
    int *pend0a = nullptr, *pend0b = nullptr, *pend1a = nullptr, *pend1b = nullptr;
    int npending = 0;
    auto publish = [&]() {
      if (npending == 0) return;
      fence_proxy_async_global();   // generic-proxy stores -> other CTAs' TMA reads
      __threadfence();
      __syncwarp();
      if (lane == 0) {
        atomicAdd(pend0a, 1);
        if (pend0b) atomicAdd(pend0b, 1);
        if (npending > 1) {
          atomicAdd(pend1a, 1);
          if (pend1b) atomicAdd(pend1b, 1);
        }
      }
      npending = 0;
    };
    // publish before blocking on a barrier that is not yet complete (warp-uniform)
    auto publish_if_blocked = [&](uint64_t* bar, uint32_t parity) {
      if (npending > 0 && __any_sync(0xffffffffu, !ptx::mbar_test_wait(bar, parity))) publish();
    };
    int acc = 0;
    uint32_t aph = 0;
    for (int i = 0;; ++i) {
      const int slot = i % kTileRing;
      const uint32_t tpar = (i / kTileRing) & 1;
      publish_if_blocked(&tile_full[slot], tpar);
      // every wait result is made warp-uniform: the warp then leaves together (the
      // TMEM loads below are warp-collective)
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&tile_full[slot], tpar, abort_flag, args.wait_ns))) {
        fail();
        break;
      }
      const TileSlot ts = tile_ring[slot];
      if (ts.t < 0) break;
      const PhaseArgs& P = args.ph[ts.phase];
      const int rows = ts.rows;
      const int row0 = ts.row0;
      const int feat0 = ts.mt * kBM + q * 32;      // first feature of this warp
      const int f = feat0 + lane;
      // operands of the epilogue, fetched before the accumulator is ready:
      // this lane's bias, and the destination row / gate of column (c0 + lane)
      // of each of this warp's column chunks
      constexpr int kMaxChunks = 256 / 64;         // chunks of 32 per warp at 256 rows
      const float bias = (f < P.M) ? __bfloat162float(P.bias[(size_t)ts.e * P.a_rows + f]) : 0.f;
      const bool glu = kGlu && ts.phase == 0;
      float bias_v = 0.f;
      if constexpr (kGlu) {
        if (glu && f < P.M) bias_v = __bfloat162float(P.bias[(size_t)ts.e * P.a_rows + P.M + f]);
      }
      int dsts[kMaxChunks];
      float gs[kMaxChunks];
#pragma unroll
      for (int k = 0; k < kMaxChunks; ++k) {
        const int col = (2 * k + half) * 32 + lane;
        if (P.mode == 1) {
          dsts[k] = (col < rows) ? __ldg(args.slot_token + row0 + col) : 0;
        } else {
          dsts[k] = row0 + col;
        }
        if (col < rows && !checked_index(dsts[k] >= 0 && dsts[k] < args.T_rows, args.err))
          dsts[k] = 0;
      }
#pragma unroll
      for (int k = 0; k < kMaxChunks; ++k) {
        const int col = (2 * k + half) * 32 + lane;
        gs[k] = (P.mode == 1 && col < rows) ? __ldg(args.gate + dsts[k]) : 1.f;
      }
      publish_if_blocked(&tfull_bar[acc], aph);
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&tfull_bar[acc], aph, abort_flag, args.wait_ns))) {
        fail();
        break;
      }
      ptx::tc_fence_after();
      const uint32_t t_base =
          tmem_base + static_cast<uint32_t>(acc * acc_cols) + (static_cast<uint32_t>(q * 32) << 16);
      if (kSplit && ts.grp >= 0) {
        // GEMM2 sub-tile of a split: the fp32 partial of this warp's 32
        // features and column chunks goes to partial tile ks of the group, as
        // [token column][feature] rows (a warp's stores cover 128 contiguous
        // bytes); the reduce kernel finishes the tile
        float* pt = args.part + (static_cast<size_t>(ts.grp) * ts.nsplit + ts.ks) * args.bn * kBM +
                    q * 32 + lane;
#pragma unroll
        for (int k = 0; k < kMaxChunks; ++k) {
          const int c0 = (2 * k + half) * 32;
          if (c0 >= rows) break;
          uint32_t r[32];
          ptx::tmem_ld_32x32b_x32(t_base + static_cast<uint32_t>(c0), r);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j < rows) pt[static_cast<size_t>(c0 + j) * kBM] = __uint_as_float(r[j]);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(&tempty_bar[acc]);
          ptx::mbar_arrive(&tile_empty[slot]);
        }
        if (++acc == args.num_acc) { acc = 0; aph ^= 1u; }
        continue;
      }
#pragma unroll
      for (int k = 0; k < kMaxChunks; ++k) {
        const int c0 = (2 * k + half) * 32;
        if (c0 >= rows) break;
        const int dst = dsts[k];
        const float g = gs[k];
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(t_base + static_cast<uint32_t>(c0), r);
        bool stored = false;
        if constexpr (kGlu) {
          if (glu) {
            // GELU(gate) * value, the value accumulator in the upper half
            uint32_t rv[32];
            ptx::tmem_ld_32x32b_x32(t_base + static_cast<uint32_t>(acc_cols / 2 + c0), rv);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float gt = __uint_as_float(r[j]) + bias;
              const float vl = __uint_as_float(rv[j]) + bias_v;
              const float h = 0.5f * gt * (1.0f + erff(gt * 0.70710678118654752f)) * vl;
              st[j * 32 + lane] = __float2bfloat16_rn(h);
            }
            stored = true;
          }
        }
        if (!stored) {
          ptx::tmem_ld_wait();
          const bool relu = P.mode == 0;
#pragma unroll
          for (int j = 0; j < 32; j += 2) {   // two tokens per conversion
            float v0 = __uint_as_float(r[j]) + bias, v1 = __uint_as_float(r[j + 1]) + bias;
            if (relu) {
              v0 = fmaxf(v0, 0.f);
              v1 = fmaxf(v1, 0.f);
            } else {
              v0 *= __shfl_sync(0xffffffffu, g, j);
              v1 *= __shfl_sync(0xffffffffu, g, j + 1);
            }
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
            st[j * 32 + lane] = h2.x;
            st[(j + 1) * 32 + lane] = h2.y;
          }
        }
        __syncwarp();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int idx = lane + 32 * kk;
          const int j = idx >> 2, part = idx & 3;
          const int drow = __shfl_sync(0xffffffffu, dst, j);
          if (c0 + j < rows && feat0 + part * 8 < P.M) {
            *reinterpret_cast<uint4*>(P.out + (size_t)drow * P.M + feat0 + part * 8) =
                *reinterpret_cast<const uint4*>(st + j * 32 + part * 8);
          }
        }
        __syncwarp();
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&tempty_bar[acc]);
        ptx::mbar_arrive(&tile_empty[slot]);
      }
      if (ts.phase == 0) {
        if (npending == 0) {
          pend0a = ts.rdy0;
          pend0b = ts.rdy1;
        } else {
          pend1a = ts.rdy0;
          pend1b = ts.rdy1;
        }
        if (++npending == kMaxPending) publish();
      }
      if (++acc == args.num_acc) { acc = 0; aph ^= 1u; }
    }
    publish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kTmemCols);
  }
}

// The split GEMM2 tiles, finished: one thread per 4 features of one token
// column of a group (an expert's 128 features by one token tile; a warp covers
// one column, so each partial is read as 512 contiguous bytes).  Block b takes
// items [256 * (b % parts), ...) of group b / parts (parts = bn * 32 / 256).  The
// partials are added in k order (deterministic), then the bias, the token's
// gate and the bf16 store to the token's output row.  Launched after the FFN
// (programmatic dependency).
constexpr int kReduceThreads = 256;
__global__ void __launch_bounds__(kReduceThreads)
ffn_split_reduce_kernel(const float* __restrict__ part, const int4* __restrict__ groups,
                        const int* __restrict__ exp_rows, const int* __restrict__ exp_base,
                        const int* __restrict__ slot_token, const float* __restrict__ gate,
                        const __nv_bfloat16* __restrict__ b2, __nv_bfloat16* __restrict__ out,
                        int S, int bn, int M, int T_rows, int* err) {
  pdl_trigger();
  pdl_wait();   // the partial tiles and the group table come from earlier kernels
  const int parts = bn * (kBM / 4) / kReduceThreads;
  const int grp = blockIdx.x / parts;
  const int item = (blockIdx.x % parts) * kReduceThreads + threadIdx.x;
  const int4 gd = groups[grp];
  if (gd.x < 0) return;
  const int e = gd.x, mt = gd.y, nt = gd.z;
  const int col = item / (kBM / 4);
  const int f4 = (item % (kBM / 4)) * 4;
  const int f = mt * kBM + f4;
  const int rows = min(bn, __ldg(exp_rows + e) - nt * bn);
  if (col >= rows || f >= M) return;
  const int row0 = __ldg(exp_base + e) + nt * bn;
  int dst = __ldg(slot_token + row0 + col);
  const size_t tile = static_cast<size_t>(bn) * kBM;   // floats per partial tile
  const float* src = part + static_cast<size_t>(grp) * S * tile + static_cast<size_t>(col) * kBM + f4;
  float4 w[kSplitFactor];
#pragma unroll
  for (int ks = 0; ks < kSplitFactor; ++ks)   // every partial in flight at once
    if (ks < S) w[ks] = __ldcg(reinterpret_cast<const float4*>(src + ks * tile));
  if (!checked_index(dst >= 0 && dst < T_rows, err)) dst = 0;
  const float g = __ldg(gate + dst);
  float4 v = w[0];
#pragma unroll
  for (int ks = 1; ks < kSplitFactor; ++ks) {   // added in k order
    if (ks < S) {
      v.x += w[ks].x;
      v.y += w[ks].y;
      v.z += w[ks].z;
      v.w += w[ks].w;
    }
  }
  const __nv_bfloat16* bb = b2 + static_cast<size_t>(e) * M + f;
  const float o0 = (v.x + __bfloat162float(bb[0])) * g;
  const float o1 = (v.y + __bfloat162float(bb[1])) * g;
  const float o2 = (v.z + __bfloat162float(bb[2])) * g;
  const float o3 = (v.w + __bfloat162float(bb[3])) * g;
  __nv_bfloat162 lo2 = __floats2bfloat162_rn(o0, o1), hi2 = __floats2bfloat162_rn(o2, o3);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&lo2);
  pk.y = *reinterpret_cast<uint32_t*>(&hi2);
  *reinterpret_cast<uint2*>(out + static_cast<size_t>(dst) * M + f) = pk;
}

size_t ffn_smem_bytes(int bn, int stages, int cached_prefix_ints, int a_tiles = 1) {
  return 1024 + static_cast<size_t>(cached_prefix_ints) * sizeof(int) +
         static_cast<size_t>(stages) * (a_tiles * kABytes + static_cast<size_t>(bn) * kBK * 2) +
         kEpiStageBytes + (2 * kMaxStages + 2 * kMaxAcc + 2 + 2 * kTileRing) * sizeof(uint64_t) +
         kTileRing * sizeof(TileSlot) + 2 * sizeof(uint32_t);
}

}  // namespace

int bf16_tile_rows(int64_t C_eff) {
  int64_t r = (C_eff + 15) / 16 * 16;
  if (r < 16) r = 16;
  if (r > 256) r = 256;
  return static_cast<int>(r);
}

cudaError_t launch_expert_ffn_bf16(const Shape& s, const Workspace& ws, const CUtensorMap& tmA1,
                                   const CUtensorMap& tmB1, const CUtensorMap& tmA2,
                                   const CUtensorMap& tmB2, const void* b1, const void* b2,
                                   const float* gate, void* out, int num_sms,
                                   cudaStream_t stream) {
  constexpr size_t kMaxSmem = 232448;   // 227 KiB opt-in per block
  FfnArgs a;
  a.tile_prefix = ws.tile_prefix;
  a.exp_rows = ws.exp_rows;
  a.exp_base = ws.exp_base;
  a.gate = gate;
  a.slot_token = ws.slot_token;
  a.ready = ws.ready;
  a.next_tile = &ws.hdr->next_tile;
  a.err = &ws.hdr->err;
  a.split = s.ffn_split;
  a.tile_prefix2 = ws.tile_prefix2;
  a.split_base = ws.split_base;
  a.part = ws.part;
  a.split_ready = ws.split_ready;
  // token-tile order within an expert when its weights sit in L2 anyway
  a.tok_major = s.d * s.d_ff * 2 * (s.glu ? 2 : 1) <= (int64_t{32} << 20) ? 1 : 0;
  a.wait_ns = wait_limit_ns();
  a.stall_test = stall_test_enabled() ? 1 : 0;
  a.num_experts = static_cast<int>(s.N);
  a.T_rows = static_cast<int>(packed_rows(s));   // packed rows; top-2 writes per assignment
  a.bn = s.tile_rows;
  a.glu = s.glu ? 1 : 0;
  if (a.glu) {
    int cols = 128;
    while (cols < 2 * a.bn) cols *= 2;          // gate and value halves of one accumulator
    a.num_acc = kTmemCols / cols;
  } else {
    a.num_acc = a.bn <= kTmemCols / kMaxAcc ? kMaxAcc : 2;
  }
  for (int p = 0; p < 2; ++p) {
    const int64_t M = p == 0 ? s.d_ff : s.d;
    const int64_t K = p == 0 ? s.d : s.d_ff;
    a.ph[p].bias = static_cast<const __nv_bfloat16*>(p == 0 ? b1 : b2);
    a.ph[p].out = static_cast<__nv_bfloat16*>(p == 0 ? ws.hbuf : out);
    a.ph[p].M = static_cast<int>(M);
    a.ph[p].a_rows = static_cast<int>(p == 0 && a.glu ? 2 * M : M);
    a.ph[p].m_tiles = static_cast<int>((M + kBM - 1) / kBM);
    a.ph[p].k_blocks = static_cast<int>((K + kBK - 1) / kBK);
    a.ph[p].mode = p == 0 ? 0 : (gate != nullptr ? 1 : 2);
  }
  const int a_tiles = a.glu ? 2 : 1;
  int stages = kMaxStages;
  while (stages > 2 && ffn_smem_bytes(a.bn, stages, 0, a_tiles) > kMaxSmem) --stages;
  a.stages = stages;
  // the tile prefix goes to shared memory when it fits beside the stage ring
  const int prefix_ints = static_cast<int>(s.N) + 1;
  a.cache_prefix = ffn_smem_bytes(a.bn, stages, prefix_ints, a_tiles) <= kMaxSmem ? 1 : 0;
  const size_t smem = ffn_smem_bytes(a.bn, stages, a.cache_prefix ? prefix_ints : 0, a_tiles);
  if (a.glu && a.split > 1) return cudaErrorInvalidValue;   // no such instantiation
  auto kern = a.glu ? expert_ffn_sm100_kernel<true, false>
                    : (a.split > 1 ? expert_ffn_sm100_kernel<false, true>
                                   : expert_ffn_sm100_kernel<false, false>);
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  err = launch_dependent(kern, dim3(num_sms), dim3(kThreads), smem, stream, tmA1, tmB1, tmA2,
                         tmB2, a);
  count_launch();
  if (err != cudaSuccess || a.split <= 1) return err;
  if (a.split > kSplitFactor || (a.bn * (kBM / 4)) % kReduceThreads != 0)
    return cudaErrorInvalidValue;
  const unsigned parts = static_cast<unsigned>(a.bn * (kBM / 4) / kReduceThreads);
  err = launch_dependent(ffn_split_reduce_kernel, dim3(kSplitMaxGroups * parts),
                         dim3(kReduceThreads), 0, stream, static_cast<const float*>(ws.part),
                         static_cast<const int4*>(static_cast<const void*>(ws.split_grp)),
                         ws.exp_rows, ws.exp_base, ws.slot_token, gate,
                         static_cast<const __nv_bfloat16*>(b2), static_cast<__nv_bfloat16*>(out),
                         a.split, a.bn, a.ph[1].M, a.T_rows, &ws.hdr->err);
  count_launch();
  return err;
}

}  // namespace swl
