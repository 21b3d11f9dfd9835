// fp32 router of the Switch layer on the 5th-generation tensor cores, for bf16
// layers: fused routing for N <= 128 experts, logits only for wider layers.
//
// The router computes z_t = W_r x_t (+ b_r) in float32, then p_t = softmax(z_t),
// e_t = argmax_i p_t,i (lowest index on ties) and g_t = p_t,e_t (Switch
// Transformer, explained, recipe step 2 "Route in float32"; paper-graph summary
// of arXiv 2101.03961, "The selective precision solution").
//
// float32 logits from bf16 tensor-core products: every fp32 router weight is
// split exactly into three bf16 numbers, w = hi + mid + lo with
//   hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid)
// (each residual is exact in fp32, and 3 x 8 significand bits cover fp32's 24).
// The layer input x is bf16 already, so every product x_k * piece_k is exact in
// fp32 and the tensor core accumulates the three dot products in fp32 (TMEM).
// z = D_hi + (D_mid + D_lo) is then the fp32 dot product up to the rounding of
// the fp32 accumulation, the same class of error as an fp32 FFMA loop.
//
// router_wsplit_kernel writes the pieces once per call, W3 = [hi; mid; lo] as a
// bf16 [3N, d] matrix; the router kernel then streams them with TMA.
//
// Fused routing (N <= 128): one cluster of S CTAs (S = 1, 2 or 4, along z) owns
// a tile of 128 tokens; CTA r takes k-blocks [r*kb_per, (r+1)*kb_per).
//   warp 0       TMA producer: x tile [128 tokens x 64 k] and the three piece
//                tiles [NP experts x 64 k] (bf16, 128-byte swizzle) per stage
//   warp 1       MMA issuer: the three piece tiles lie contiguous in shared
//                memory, one B operand of 3*NP rows; per 16-wide k step one
//                tcgen05.mma (M = 128 tokens, N = 3*NP; two MMAs when 3*NP >
//                256) into the three TMEM accumulators [hi | mid | lo]
//   warp 2       TMEM allocator
//   warp 3       stages the bias row in shared memory (-inf in padded columns)
//   warps 4..7   TMEM epilogue (thread = token row): z = D_hi + (D_mid + D_lo),
//                plus the bias when the tile has one CTA (S = 1)
// For S > 1 the partial logits of the cluster are added in rank order through
// distributed shared memory (deterministic), plus the bias.  Each CTA then
// routes its 128/S rows with all 256 threads (softmax, argmax, block ranks,
// per-expert counts and sums of p).
// Every mbarrier wait is bounded; a stuck pipeline sets the device error word.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "router_common.cuh"
#include "sm100_ptx.cuh"

namespace cg = cooperative_groups;

namespace swl {
namespace {

constexpr int kThreads = 256;
constexpr int kBM = 128;          // tokens per tile (UMMA M)
constexpr int kBK = 64;           // k per stage (one 128-byte swizzle row of bf16)
constexpr int kUmmaK = 16;
constexpr int kPieces = 3;        // hi, mid, lo
constexpr int kMaxStages = 4;
constexpr int kXAhead = 4;        // x k-blocks requested into L2 beyond the stage ring
constexpr size_t kMaxDynSmem = 232448 - 8192;   // leave room for the static arrays

template <int NP>
struct TcCfg {
  static constexpr uint32_t kABytes = kBM * kBK * 2;             // x tile, bf16
  static constexpr uint32_t kPieceBytes = NP * kBK * 2;          // one piece tile, bf16
  static constexpr uint32_t kStage = kABytes + kPieces * kPieceBytes;
  static constexpr uint32_t kTmemCols = 3 * NP <= 128 ? 128 : (3 * NP <= 256 ? 256 : 512);
};

struct TcArgs {
  const float* b_r;       // [N] or null
  float* logits;          // wide layout only: [T, N] fp32 logits (without the bias)
  int T, N;
  int piece_rows;         // rows of one piece in W3 (= N)
  int nkb;                // k-blocks of 64 over d
  int kb_per;             // k-blocks per cluster rank
  int stages;
  int* expert_idx;
  float* gate;
  int* local_rank;
  int* blk_count;
  float* blk_psum;
  WsHeader* hdr;
  unsigned long long wait_ns;   // bound of every wait
  const uint8_t* pf;      // bytes fetched into L2 once this CTA's loads have landed
  size_t pf_bytes;        // (the expert weights the FFN streams first; 0: none)
};

__device__ __forceinline__ uint32_t bf16_bits(__nv_bfloat16 h) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(h));
}

// w = hi + mid + lo exactly (see the file comment).
__device__ __forceinline__ void split3(float w, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(w);
  const float r1 = w - __bfloat162float(h);
  const __nv_bfloat16 m = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(m);
  hi = bf16_bits(h);
  mid = bf16_bits(m);
  lo = bf16_bits(__float2bfloat16_rn(r2));
}

// W3[p*N + n, k] = piece p of W_r[n, k]; 8 consecutive k per thread (d % 8 == 0).
__global__ void __launch_bounds__(256)
router_wsplit_kernel(const float* __restrict__ W_r, __nv_bfloat16* __restrict__ W3, int N, int d) {
  pdl_trigger();
  const size_t chunks = static_cast<size_t>(N) * (d / 8);
  const size_t plane = static_cast<size_t>(N) * d;
  for (size_t c = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; c < chunks;
       c += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t off = c * 8;
    const float4 u0 = *reinterpret_cast<const float4*>(W_r + off);
    const float4 u1 = *reinterpret_cast<const float4*>(W_r + off + 4);
    const float w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    uint32_t hi[4], mi[4], lo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t h0, m0, l0, h1, m1, l1;
      split3(w[2 * q], h0, m0, l0);
      split3(w[2 * q + 1], h1, m1, l1);
      hi[q] = h0 | (h1 << 16);
      mi[q] = m0 | (m1 << 16);
      lo[q] = l0 | (l1 << 16);
    }
    *reinterpret_cast<uint4*>(W3 + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(W3 + plane + off) = make_uint4(mi[0], mi[1], mi[2], mi[3]);
    *reinterpret_cast<uint4*>(W3 + 2 * plane + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// Fused routing of N <= NP experts (cluster of S CTAs along z).
template <int NP>
__global__ void __launch_bounds__(kThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const TcArgs a) {
  // tmW: W3 = [hi; mid; lo] as bf16 [3N, d], box [NP rows, 64 k], 128-byte swizzle
  using C = TcCfg<NP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = a.stages;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + stages * C::kStage);
  uint64_t* empty_bar = full_bar + kMaxStages;
  uint64_t* accf_bar = empty_bar + kMaxStages;
  uint64_t* drain_bar = accf_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* Ps = reinterpret_cast<float*>(smem);   // [kBM][PS] logits, after the main loop
  __shared__ int eid[kBM];
  __shared__ int wcnt[(kBM / 32) * NP];
  __shared__ float red[256];
  __shared__ float bias_s[NP];   // b_r, 0 without a bias, -inf in the padded columns

  cg::cluster_group cluster = cg::this_cluster();
  const int S = static_cast<int>(cluster.num_blocks());
  const int r = static_cast<int>(cluster.block_rank());
  // row stride of the logits tile: NP + 2S (= NP + threads per token in the
  // routing below, so that a warp's reads fall in distinct banks)
  const int PS = NP + 2 * S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  if (blockIdx.x == 0 && blockIdx.y == 0 && r == 0 && threadIdx.x == 0) {
    a.hdr->err = kDevOk;   // per-call device status
    a.hdr->done = 0u;      // arrival counter of the dispatch scan
  }
  const int m0 = static_cast<int>(blockIdx.x) * kBM;
  constexpr int n0 = 0;
  const int kb0 = r * a.kb_per;
  const int nk = max(0, min(a.nkb, kb0 + a.kb_per) - kb0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(&full_bar[s], 1);
      ptx::mbar_init(&empty_bar[s], 1);
    }
    ptx::mbar_init(accf_bar, 1);
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tmap(&tmX);
    ptx::prefetch_tmap(&tmW);
  }
  if (warp == 2) {
    ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(&a.hdr->err, kDevPipelineTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_x = ptx::l2_policy_evict_last();    // x: the gather reads it again
      const uint64_t pol_w = ptx::l2_policy_evict_last();    // W3: read by every tile
      uint32_t issued = 0u, last_par = 0u;
      // x does not depend on the split kernel: the first stages' x tiles are
      // requested before waiting for it, then their W3 pieces
      const int first = nk < stages ? nk : stages;
      for (int i = 0; i < first; ++i) {
        ptx::mbar_arrive_expect_tx(&full_bar[i], C::kStage);
        ptx::tma_load_2d(smem + i * C::kStage, &tmX, &full_bar[i], (kb0 + i) * kBK, m0, pol_x);
        issued |= 1u << i;
      }
      // x comes from HBM: its next kXAhead k-blocks beyond the stage ring are
      // requested into L2 ahead of their TMA loads (more bytes in flight than
      // the stages' shared memory holds)
      for (int i = first; i < nk && i < first + kXAhead; ++i)
        ptx::tma_prefetch_2d(&tmX, (kb0 + i) * kBK, m0);
      pdl_wait();   // W3 comes from the split kernel
      for (int i = 0; i < nk; ++i) {
        const int s = i % stages;
        const uint32_t ph = static_cast<uint32_t>(i / stages) & 1u;
        uint8_t* st = smem + s * C::kStage;
        const int kc = (kb0 + i) * kBK;
        if (i >= first) {
          if (!ptx::mbar_wait(&empty_bar[s], ph ^ 1u, abort_flag, a.wait_ns)) {
            fail();
            break;
          }
          ptx::mbar_arrive_expect_tx(&full_bar[s], C::kStage);
          ptx::tma_load_2d(st, &tmX, &full_bar[s], kc, m0, pol_x);
          if (i + kXAhead < nk) ptx::tma_prefetch_2d(&tmX, (kb0 + i + kXAhead) * kBK, m0);
        }
#pragma unroll
        for (int p = 0; p < kPieces; ++p)
          ptx::tma_load_2d(st + C::kABytes + p * C::kPieceBytes, &tmW, &full_bar[s], kc,
                           p * a.piece_rows + n0, pol_w);
        issued |= 1u << s;
        last_par = (last_par & ~(1u << s)) | (ph << s);
      }
      // every issued load lands before the stage memory is reused or the CTA exits
      for (int s = 0; s < stages; ++s) {
        if (issued & (1u << s)) {
          volatile int never = 0;
          if (!ptx::mbar_wait(&full_bar[s], (last_par >> s) & 1u, &never, a.wait_ns))
            atomicExch(&a.hdr->err, kDevPipelineTimeout);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // the three piece tiles are contiguous in shared memory: one operand of
      // 3*NP rows, issued as MMAs of at most 256 rows (N <= 256)
      constexpr int kRows = kPieces * NP;
      constexpr int kChunks = (kRows + 255) / 256;
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        const int s = i % stages;
        const uint32_t ph = static_cast<uint32_t>(i / stages) & 1u;
        if (!ptx::mbar_wait(&full_bar[s], ph, abort_flag, a.wait_ns)) {
          fail();
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a_addr = ptx::smem_u32(smem + s * C::kStage);
        const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
        for (int k = 0; k < kBK / kUmmaK; ++k) {
          const uint64_t ad = ptx::umma_desc_sw128_kmajor(a_addr + k * kUmmaK * 2);
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            constexpr uint32_t kRowBytes = kBK * 2;
            const uint32_t n = kRows - c * 256 < 256 ? kRows - c * 256 : 256;
            const uint64_t bd = ptx::umma_desc_sw128_kmajor(b_addr + c * 256 * kRowBytes +
                                                            k * kUmmaK * 2);
            ptx::umma_bf16(tmem_base + static_cast<uint32_t>(c * 256), ad, bd,
                           ptx::umma_idesc_bf16_f32(n), (i | k) != 0 ? 1u : 0u);
          }
        }
        ptx::umma_commit(&empty_bar[s]);    // frees the stage once these MMAs are done
      }
      if (ok && nk > 0) ptx::umma_commit(accf_bar);
      // all MMAs of this thread complete before TMEM is released
      ptx::umma_commit(drain_bar);
      volatile int never = 0;
      if (!ptx::mbar_wait(drain_bar, 0u, &never, a.wait_ns)) atomicExch(&a.hdr->err, kDevPipelineTimeout);
    }
    __syncwarp();
  } else if (warp == 3) {
    // bias row for the read-out below (named barrier 1: this warp + warps 4..7)
    for (int n = lane; n < NP; n += 32)
      bias_s[n] = n < a.N ? (a.b_r ? a.b_r[n] : 0.f) : -INFINITY;
    ptx::named_bar_arrive(1, 160);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ TMEM epilogue
    bool have = false;
    if (nk > 0) {
      const bool got = ptx::mbar_wait(accf_bar, 0u, abort_flag, a.wait_ns);
      have = __all_sync(0xffffffffu, got);
      if (!have && lane == 0) fail();
    }
    ptx::named_bar_sync(1, 160);
    // a lone CTA (S = 1) holds the whole sum: the bias goes in here
    const bool add_bias = S == 1;
    ptx::tc_fence_after();
    const int q = warp & 3;
    const int row = q * 32 + lane;                 // TMEM lane = token row of the tile
#pragma unroll 1
    for (int c0 = 0; c0 < NP; c0 += 32) {
      float z[32];
      if (have) {
        uint32_t r0[32], r1[32], r2[32];
        const uint32_t ta = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                            static_cast<uint32_t>(c0);
        ptx::tmem_ld_32x32b_x32(ta, r0);
        ptx::tmem_ld_32x32b_x32(ta + NP, r1);
        ptx::tmem_ld_32x32b_x32(ta + 2 * NP, r2);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          z[j] = __uint_as_float(r0[j]) + (__uint_as_float(r1[j]) + __uint_as_float(r2[j]));
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) z[j] = 0.f;
      }
      if (add_bias) {
#pragma unroll
        for (int j = 0; j < 32; ++j) z[j] = c0 + j < a.N ? z[j] + bias_s[c0 + j] : -INFINITY;
      }
      float* pr = Ps + row * PS + c0;
      if ((PS & 3) == 0) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(pr + j) = make_float4(z[j], z[j + 1], z[j + 2], z[j + 3]);
      } else {   // PS = NP + 2: rows 8-byte aligned
#pragma unroll
        for (int j = 0; j < 32; j += 2)
          *reinterpret_cast<float2*>(pr + j) = make_float2(z[j], z[j + 1]);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, C::kTmemCols);
  }
  // this CTA's rows [r*R, r*R + R), with the bias added and -inf in the padded
  // columns (S > 1: written in place, the peers read only their own rows of
  // this tile; S = 1: added by the read-out above)
  const int R = kBM / S;
  const int row0 = r * R;
  if (S > 1) {
    cluster.sync();   // every partial logits tile of the cluster is complete
    // partials added in rank order (PS = NP + 2S is a multiple of 4 here)
    const float* part[4];
#pragma unroll
    for (int s2 = 0; s2 < 4; ++s2) part[s2] = cluster.map_shared_rank(Ps, s2 < S ? s2 : 0);
    for (int idx = threadIdx.x; idx < R * (NP / 4); idx += kThreads) {
      const int i = idx / (NP / 4), n = (idx % (NP / 4)) * 4;
      const int off = (row0 + i) * PS + n;
      float4 v = *reinterpret_cast<const float4*>(part[0] + off);
#pragma unroll
      for (int s2 = 1; s2 < 4; ++s2) {
        if (s2 < S) {
          const float4 u = *reinterpret_cast<const float4*>(part[s2] + off);
          v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
        }
      }
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int c = 0; c < 4; ++c)
        Ps[off + c] = (n + c < a.N) ? vv[c] + bias_s[n + c] : -INFINITY;
    }
    cluster.sync();   // the peers have finished reading this CTA's partial tile
  }

  const int t0 = m0 + row0;
  const int ntok = max(0, min(R, a.T - t0));
  const int blk = blockIdx.x * S + r;
  if (S == 1)
    route_rows_grouped<NP, 128>(Ps, PS, ntok, t0, a.N, blk, a.expert_idx, a.gate, a.local_rank,
                                a.blk_count, a.blk_psum, a.hdr, eid, wcnt, red);
  else if (S == 2)
    route_rows_grouped<NP, 64>(Ps + row0 * PS, PS, ntok, t0, a.N, blk, a.expert_idx, a.gate,
                               a.local_rank, a.blk_count, a.blk_psum, a.hdr, eid, wcnt, red);
  else
    route_rows_grouped<NP, 32>(Ps + row0 * PS, PS, ntok, t0, a.N, blk, a.expert_idx, a.gate,
                               a.local_rank, a.blk_count, a.blk_psum, a.hdr, eid, wcnt, red);
  // HBM is idle from here until the expert FFN starts (every CTA's loads have
  // landed by now): this CTA's share of the weights the FFN streams first goes
  // to L2 meanwhile (no completion needed).  Issued last, so that no warp of
  // the routing above waits for it.
  if (threadIdx.x == 0 && a.pf_bytes > 0) {
    constexpr size_t kChunk = 64 << 10;
    const size_t nct = static_cast<size_t>(gridDim.x) * gridDim.y * gridDim.z;
    const size_t id = (static_cast<size_t>(blockIdx.z) * gridDim.y + blockIdx.y) * gridDim.x +
                      blockIdx.x;
    const size_t share = ((a.pf_bytes + nct - 1) / nct + 15) & ~static_cast<size_t>(15);
    const size_t lo = id * share;
    const size_t hi = lo + share < a.pf_bytes ? lo + share : a.pf_bytes;
    for (size_t o = lo; o < hi; o += kChunk) {
      const size_t n = (hi - o < kChunk ? hi - o : kChunk) & ~static_cast<size_t>(15);
      if (n > 0) ptx::prefetch_l2_bulk(a.pf + o, static_cast<uint32_t>(n));
    }
  }
}

// Logits of wide layers (N > 128 experts), persistent: one CTA per SM takes
// units u = blockIdx.x, blockIdx.x + gridDim.x, ... of kTT token tiles of 128
// tokens by one tile of 128 experts (expert tiles fastest, so the CTAs running
// together share x tiles in L2; W3 stays in L2), and writes them to a.logits
// [T, N] fp32 without the bias (the softmax kernel adds it).
//   warp 0       TMA producer: per k-block the unit's x tiles and the three W
//                piece tiles into a ring of stages, across units
//   warp 1       MMA issuer: per 16-wide k step and token tile, x * hi, x * mid
//                and x * lo into the tile's accumulator (128 TMEM columns)
//   warp 2       TMEM allocator (512 columns: 512 / (128 kTT) unit accumulators)
//   warps 4..    read-out, four warps per token tile (thread = token row): z,
//                32 experts at a time, transposed through shared memory into
//                row-major 128-byte stores
// Each product x_k * piece_k is exact, and all of them go into one fp32
// accumulator: 3 x 64 tensor-core accumulation steps of a 1024-wide row
// against 1024 roundings of an fp32 FFMA loop.  kTT = 2: the W pieces of a
// k-block serve two token tiles (80 KB of operands per two tiles instead of
// 128); with one 128-column accumulator per token tile, two units fit in TMEM
// and a unit's read-out runs under the next unit's MMAs.
// kXP = 3: the router input is itself three bf16 pieces (a jittered fp32
// input, x3 = [xh; xm; xl] [3T, d]); per k step six MMAs keep every product
// above fp32's resolution: xh wh, xh wm, xh wl, xm wh, xm wm and xl wh (xm wl,
// xl wm and xl wl are below 2^-24 of the result).
constexpr int kWideNP = 128;          // experts per tile
constexpr int kWidePitch = 33;        // transpose tile row pitch (floats)
using WideCfg = TcCfg<kWideNP>;

template <int kXP, int kTT>
struct WideK {
  static constexpr uint32_t kXB = kTT * kXP * WideCfg::kABytes;      // x bytes of a stage
  static constexpr uint32_t kStageB = kXB + kPieces * WideCfg::kPieceBytes;
  static constexpr int kSt = kStageB <= 64 * 1024 ? 3 : 2;
  static constexpr int kAccCols = kTT * kWideNP;                     // TMEM columns of a unit
  static constexpr int kBufs = 512 / kAccCols;
  static constexpr int kEpiWarps = 4 * kTT;
  static constexpr int kThreads = 128 + 32 * kEpiWarps;
  static constexpr size_t kBarOff = static_cast<size_t>(kSt) * kStageB;
  static constexpr size_t kStgOff = kBarOff + 256;
  static constexpr size_t kSmem =
      1024 + kStgOff + static_cast<size_t>(kEpiWarps) * 32 * kWidePitch * sizeof(float);
  static_assert(kSmem <= 232448, "shared memory of the wide logits kernel");
};
constexpr int kWideTT = 2;            // token tiles per unit of the plain (unjittered) input

template <int kXP, int kTT>
__global__ void __launch_bounds__(WideK<kXP, kTT>::kThreads, 1)
router_logits_wide_kernel(const __grid_constant__ CUtensorMap tmX,
                          const __grid_constant__ CUtensorMap tmW, const TcArgs a) {
  using K = WideK<kXP, kTT>;
  constexpr int kSt = K::kSt;
  // tmW: W3 = [hi; mid; lo] as bf16 [3N, d], box [128 rows, 64 k], 128-byte swizzle
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + K::kBarOff);
  uint64_t* empty_bar = full_bar + kSt;
  uint64_t* tfull = empty_bar + kSt;
  uint64_t* tempty = tfull + K::kBufs;
  uint64_t* drain_bar = tempty + K::kBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* stg = reinterpret_cast<float*>(smem + K::kStgOff);   // [epilogue warps][32][kWidePitch]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    a.hdr->err = kDevOk;   // per-call device status
    a.hdr->done = 0u;      // arrival counter of the dispatch scan
  }
  const int n_tiles = (a.N + kWideNP - 1) / kWideNP;
  const int t_tiles = (a.T + kBM - 1) / kBM;
  const int total = n_tiles * ((t_tiles + kTT - 1) / kTT);   // units
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      ptx::mbar_init(&full_bar[s], 1);
      ptx::mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < K::kBufs; ++b) {
      ptx::mbar_init(&tfull[b], 1);
      ptx::mbar_init(&tempty[b], K::kEpiWarps);   // one arrive per read-out warp
    }
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tmap(&tmX);
    ptx::prefetch_tmap(&tmW);
  }
  if (warp == 2) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(&a.hdr->err, kDevPipelineTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_x = ptx::l2_policy_evict_first();   // x: read by one row of units
      const uint64_t pol_w = ptx::l2_policy_evict_last();    // W3: read by every unit
      uint32_t issued = 0u, last_par = 0u;
      pdl_wait();   // W3 comes from the split kernel (and x3 from the jitter kernel)
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        const int m0 = (u / n_tiles) * kTT * kBM, n0 = (u % n_tiles) * kWideNP;
        for (int kb = 0; kb < a.nkb; ++kb, ++it) {
          const int s = it % kSt;
          const uint32_t ph = static_cast<uint32_t>(it / kSt) & 1u;
          if (!ptx::mbar_wait(&empty_bar[s], ph ^ 1u, abort_flag, a.wait_ns)) {
            fail();
            ok = false;
            break;
          }
          uint8_t* st = smem + s * K::kStageB;
          ptx::mbar_arrive_expect_tx(&full_bar[s], K::kStageB);
#pragma unroll
          for (int tt = 0; tt < kTT; ++tt)
#pragma unroll
            for (int p = 0; p < kXP; ++p)
              ptx::tma_load_2d(st + (tt * kXP + p) * WideCfg::kABytes, &tmX, &full_bar[s],
                               kb * kBK, p * a.T + m0 + tt * kBM, pol_x);
#pragma unroll
          for (int p = 0; p < kPieces; ++p)
            ptx::tma_load_2d(st + K::kXB + p * WideCfg::kPieceBytes, &tmW, &full_bar[s],
                             kb * kBK, p * a.piece_rows + n0, pol_w);
          issued |= 1u << s;
          last_par = (last_par & ~(1u << s)) | (ph << s);
        }
      }
      // every issued load lands before the stage memory goes away
      for (int s = 0; s < kSt; ++s) {
        if (issued & (1u << s)) {
          volatile int never = 0;
          if (!ptx::mbar_wait(&full_bar[s], (last_par >> s) & 1u, &never, a.wait_ns))
            atomicExch(&a.hdr->err, kDevPipelineTimeout);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = ptx::umma_idesc_bf16_f32(kWideNP);
      int it = 0, uc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++uc) {
        const int buf = uc % K::kBufs;
        if (!ptx::mbar_wait(&tempty[buf], (static_cast<uint32_t>(uc / K::kBufs) & 1u) ^ 1u,
                            abort_flag, a.wait_ns)) {
          fail();
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_unit = tmem_base + static_cast<uint32_t>(buf * K::kAccCols);
        for (int kb = 0; kb < a.nkb; ++kb, ++it) {
          const int s = it % kSt;
          const uint32_t ph = static_cast<uint32_t>(it / kSt) & 1u;
          if (!ptx::mbar_wait(&full_bar[s], ph, abort_flag, a.wait_ns)) {
            fail();
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t x_addr = ptx::smem_u32(smem + s * K::kStageB);
          const uint32_t b_addr = x_addr + K::kXB;
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k) {
            const uint32_t ko = k * kUmmaK * 2;
            const uint64_t wh = ptx::umma_desc_sw128_kmajor(b_addr + ko);
            const uint64_t wm = ptx::umma_desc_sw128_kmajor(b_addr + WideCfg::kPieceBytes + ko);
            const uint64_t wl = ptx::umma_desc_sw128_kmajor(b_addr + 2 * WideCfg::kPieceBytes + ko);
            const uint32_t first = (kb | k) != 0 ? 1u : 0u;
#pragma unroll
            for (int tt = 0; tt < kTT; ++tt) {
              const uint32_t a_t = x_addr + tt * kXP * WideCfg::kABytes;
              const uint32_t d_t = d_unit + static_cast<uint32_t>(tt * kWideNP);
              const uint64_t ah = ptx::umma_desc_sw128_kmajor(a_t + ko);
              ptx::umma_bf16(d_t, ah, wh, idesc, first);
              ptx::umma_bf16(d_t, ah, wm, idesc, 1u);
              ptx::umma_bf16(d_t, ah, wl, idesc, 1u);
              if constexpr (kXP == 3) {
                const uint64_t am = ptx::umma_desc_sw128_kmajor(a_t + WideCfg::kABytes + ko);
                const uint64_t al = ptx::umma_desc_sw128_kmajor(a_t + 2 * WideCfg::kABytes + ko);
                ptx::umma_bf16(d_t, am, wh, idesc, 1u);
                ptx::umma_bf16(d_t, am, wm, idesc, 1u);
                ptx::umma_bf16(d_t, al, wh, idesc, 1u);
              }
            }
          }
          ptx::umma_commit(&empty_bar[s]);   // frees the stage once these MMAs are done
        }
        if (ok) ptx::umma_commit(&tfull[buf]);
      }
      // all MMAs of this thread complete before TMEM is released
      ptx::umma_commit(drain_bar);
      volatile int never = 0;
      if (!ptx::mbar_wait(drain_bar, 0u, &never, a.wait_ns))
        atomicExch(&a.hdr->err, kDevPipelineTimeout);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ read-out
    const int q = warp & 3;                  // TMEM lanes [32q, 32q + 32): token rows
    const int tt = (warp - 4) >> 2;          // token tile of the unit
    float* st = stg + (warp - 4) * 32 * kWidePitch;
    const bool vec = (a.N % 4) == 0;
    int uc = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++uc) {
      const int buf = uc % K::kBufs;
      const bool got = ptx::mbar_wait(&tfull[buf], static_cast<uint32_t>(uc / K::kBufs) & 1u,
                                      abort_flag, a.wait_ns);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) fail();
        break;
      }
      ptx::tc_fence_after();
      const int m0 = ((u / n_tiles) * kTT + tt) * kBM + q * 32, n0 = (u % n_tiles) * kWideNP;
      const uint32_t ta = tmem_base + static_cast<uint32_t>(buf * K::kAccCols + tt * kWideNP) +
                          (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < kWideNP / 32; ++c) {
        uint32_t r0[32];
        ptx::tmem_ld_32x32b_x32(ta + static_cast<uint32_t>(c * 32), r0);
        ptx::tmem_ld_wait();
        if (c == kWideNP / 32 - 1) {
          // the whole accumulator is in registers: the MMAs of a later unit may reuse it
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j)
          st[lane * kWidePitch + j] = __uint_as_float(r0[j]);
        __syncwarp();
        // rows of the 32 x 32 block: 8 lanes per row, 4 rows per store
        const int col = (lane & 7) * 4;
        const int n = n0 + c * 32 + col;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int row = i * 4 + (lane >> 3);
          const int tok = m0 + row;
          if (tok >= a.T || n >= a.N) continue;
          const float* src = st + row * kWidePitch + col;
          float* dst = a.logits + static_cast<size_t>(tok) * a.N + n;
          if (vec) {
            *reinterpret_cast<float4*>(dst) = make_float4(src[0], src[1], src[2], src[3]);
          } else {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
              if (n + c4 < a.N) dst[c4] = src[c4];
          }
        }
        __syncwarp();
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 512);
  }
}

template <int NP>
size_t tc_smem_bytes(int stages) {
  return 1024 + static_cast<size_t>(stages) * TcCfg<NP>::kStage +
         (2 * kMaxStages + 2) * sizeof(uint64_t) + 2 * sizeof(uint32_t);
}

// Stages of the operand ring: as many as fit, except that with more one-CTA
// tiles than SMs each CTA gets two, so that two CTAs share an SM (their shared
// memory, registers and 2 x 256 TMEM columns fit) and all tiles are resident at
// once; each CTA's prologue and routing tail then overlap the other CTA's loads
// instead of forming a second wave.
template <int NP>
int tc_stages(const Shape& s, int num_sms) {
  int stages = kMaxStages;
  while (stages > 2 && tc_smem_bytes<NP>(stages) > kMaxDynSmem) --stages;
  const int64_t t_tiles = (s.T + kBM - 1) / kBM;
  if (s.ksplit_eff == 1 && 3 * NP <= 256 && t_tiles > num_sms) stages = 2;
  return stages;
}

template <int NP>
cudaError_t launch_tc_t(const Shape& s, const Workspace& ws, const CUtensorMap& tmX,
                        const CUtensorMap& tmW, const float* b_r, int* expert_idx, float* gate,
                        int* local_rank, const void* pf, size_t pf_bytes, int num_sms,
                        cudaStream_t stream) {
  TcArgs a;
  a.pf = static_cast<const uint8_t*>(pf);
  a.pf_bytes = pf_bytes;
  a.b_r = b_r;
  a.logits = ws.logits;
  a.T = static_cast<int>(s.T);
  a.N = static_cast<int>(s.N);
  a.piece_rows = static_cast<int>(s.N);
  a.nkb = static_cast<int>((s.d + kBK - 1) / kBK);
  a.kb_per = s.kslice / kBK;
  a.expert_idx = expert_idx;
  a.gate = gate;
  a.local_rank = local_rank;
  a.blk_count = ws.blk_count;
  a.blk_psum = ws.blk_psum;
  a.hdr = ws.hdr;
  a.wait_ns = wait_limit_ns();
  const unsigned t_tiles = static_cast<unsigned>((s.T + kBM - 1) / kBM);
  const int stages = tc_stages<NP>(s, num_sms);
  // the logits tile reuses the stage memory
  const size_t ps_bytes = static_cast<size_t>(kBM) * (NP + 2 * s.ksplit_eff) * 4;
  if (ps_bytes > static_cast<size_t>(stages) * TcCfg<NP>::kStage) return cudaErrorInvalidValue;
  a.stages = stages;
  const size_t smem = tc_smem_bytes<NP>(stages);
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<NP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(t_tiles, 1, static_cast<unsigned>(s.ksplit_eff));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = static_cast<unsigned>(s.ksplit_eff);
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, router_tc_kernel<NP>, tmX, tmW, a);
}

template <int kXP, int kTT>
cudaError_t launch_wide_t(const TcArgs& a, const CUtensorMap& tmX, const CUtensorMap& tmW,
                          int64_t units, int num_sms, cudaStream_t stream) {
  using K = WideK<kXP, kTT>;
  const unsigned grid = static_cast<unsigned>(units < num_sms ? units : num_sms);
  cudaError_t e = cudaFuncSetAttribute(router_logits_wide_kernel<kXP, kTT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(K::kSmem));
  if (e != cudaSuccess) return e;
  return launch_dependent(router_logits_wide_kernel<kXP, kTT>, dim3(grid), dim3(K::kThreads),
                          K::kSmem, stream, tmX, tmW, a);
}

cudaError_t launch_wide(const Shape& s, const Workspace& ws, const CUtensorMap& tmX,
                        const CUtensorMap& tmW, int num_sms, cudaStream_t stream) {
  TcArgs a = {};
  a.logits = ws.logits;
  a.T = static_cast<int>(s.T);
  a.N = static_cast<int>(s.N);
  a.piece_rows = static_cast<int>(s.N);
  a.nkb = static_cast<int>((s.d + kBK - 1) / kBK);
  a.hdr = ws.hdr;
  a.wait_ns = wait_limit_ns();
  const int64_t t_tiles = (s.T + kBM - 1) / kBM, n_tiles = (s.N + kWideNP - 1) / kWideNP;
  if (s.xsplit) return launch_wide_t<3, 1>(a, tmX, tmW, t_tiles * n_tiles, num_sms, stream);
  return launch_wide_t<1, kWideTT>(a, tmX, tmW, (t_tiles + kWideTT - 1) / kWideTT * n_tiles,
                                   num_sms, stream);
}

}  // namespace

int router_tc_padded_experts(int64_t N) {
  return N > kFusedRouterMaxN ? 128 : static_cast<int>((N + 31) / 32 * 32);
}

int router_tc_stages(const Shape& s, int num_sms) {
  if (s.router_path == kRouterTCWide) return s.xsplit ? WideK<3, 1>::kSt : WideK<1, kWideTT>::kSt;
  switch (router_tc_padded_experts(s.N)) {
    case 32: return tc_stages<32>(s, num_sms);
    case 64: return tc_stages<64>(s, num_sms);
    case 96: return tc_stages<96>(s, num_sms);
    case 128: return tc_stages<128>(s, num_sms);
    default: return 0;
  }
}

cudaError_t launch_router_tc(const Shape& s, const Workspace& ws, const float* W_r,
                             const CUtensorMap& tmX, const CUtensorMap& tmW, const float* b_r,
                             int* expert_idx, float* gate, int* local_rank,
                             const void* l2_prefetch, size_t l2_prefetch_bytes, int num_sms,
                             cudaStream_t stream) {
  // the three bf16 pieces of W_r, then the router (programmatic dependent launch)
  const size_t chunks = static_cast<size_t>(s.N) * static_cast<size_t>(s.d / 8);
  size_t blocks = (chunks + 255) / 256;
  if (blocks > 4 * 148) blocks = 4 * 148;
  if (blocks < 1) blocks = 1;
  router_wsplit_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      W_r, static_cast<__nv_bfloat16*>(ws.w3), static_cast<int>(s.N), static_cast<int>(s.d));
  cudaError_t e = cudaGetLastError();
  count_launch();
  if (e != cudaSuccess) return e;
  if (s.router_path == kRouterTCWide) {
    e = launch_wide(s, ws, tmX, tmW, num_sms, stream);
  } else {
    switch (router_tc_padded_experts(s.N)) {
      case 32: e = launch_tc_t<32>(s, ws, tmX, tmW, b_r, expert_idx, gate, local_rank, l2_prefetch, l2_prefetch_bytes, num_sms, stream); break;
      case 64: e = launch_tc_t<64>(s, ws, tmX, tmW, b_r, expert_idx, gate, local_rank, l2_prefetch, l2_prefetch_bytes, num_sms, stream); break;
      case 96: e = launch_tc_t<96>(s, ws, tmX, tmW, b_r, expert_idx, gate, local_rank, l2_prefetch, l2_prefetch_bytes, num_sms, stream); break;
      case 128: e = launch_tc_t<128>(s, ws, tmX, tmW, b_r, expert_idx, gate, local_rank, l2_prefetch, l2_prefetch_bytes, num_sms, stream); break;
      default: e = cudaErrorInvalidValue; break;
    }
  }
  count_launch();
  return e;
}

}  // namespace swl
