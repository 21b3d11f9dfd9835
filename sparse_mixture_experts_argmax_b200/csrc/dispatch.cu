// Dispatch of the Switch layer: capacity, positions, drops and the gather into
// per-expert buffers, plus the load-balancing loss.
//
// Positions follow the cumulative sum over each expert's column of the dispatch
// mask in token order; a token whose position reaches the expert capacity
// overflows and is dropped (paper-graph summary of arXiv 2101.03961, section
// 3.4, "The routing mechanics in detail"; capacity C = ceil(cf * T / N) from
// the "Capacity Factor" section of the Switch Transformer reading note).
// Dropped tokens get a zero layer output (Switch Transformer, explained: they
// skip the expert and continue on the residual path, which is outside this layer).
//
// Aux loss = N * sum_i f_i P_i with f_i the fraction of tokens whose argmax is i
// and P_i the mean router probability of i ("The loss formulation"), returned
// without the alpha factor.
//
// dispatch_scan_kernel:   per expert, exclusive scan of the per-block counts over
//                         token blocks (token order); expert totals; fp64 sums of
//                         p.  The last CTA to finish scans over experts (packed
//                         row bases, GEMM tile prefix) and writes the aux loss.
// dispatch_gather_kernel: pos = block offset + in-block rank; kept tokens are
//                         copied into their packed row of the expert buffer with
//                         16-byte vector moves (rows requested early when x is
//                         small enough to still be in L2), dropped tokens' output
//                         rows zeroed.
// dispatch_fused_kernel:  both in one launch for N <= 128 and small batches.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "kernels.h"

namespace swl {
namespace {

constexpr int kScanThreads = 512;
constexpr int kScanWarps = kScanThreads / 32;

// Inclusive warp scan (Hillis-Steele with shuffles; fixed order, deterministic).
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += u;
  }
  return v;
}

// Exclusive scan over the block of one int per thread; returns the exclusive
// prefix and writes the block total to *total.  Uses s_warp[kScanWarps].
__device__ __forceinline__ int block_excl_scan(int v, int* s_warp, int* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int incl = warp_incl_scan(v, lane);
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < kScanWarps ? s_warp[lane] : 0;
    const int wi = warp_incl_scan(w, lane);
    if (lane < kScanWarps) s_warp[lane] = wi - w;   // exclusive warp offsets
    if (lane == kScanWarps - 1) *total = wi;
  }
  __syncthreads();
  const int r = s_warp[warp] + incl - v;
  __syncthreads();
  return r;
}

// record != nullptr (a shard of a global batch): the expert totals of this
// rank's tokens also go to the exchange record (int32 counts, then fp64 sums
// at record_psum_offset), and the expert-level part (capacity, bases, aux) is
// left to shard_combine_kernel, which needs every rank's record.
__global__ void __launch_bounds__(kScanThreads)
dispatch_scan_kernel(const int* __restrict__ blk_count, const float* __restrict__ blk_psum,
                     int* __restrict__ blk_off, int* __restrict__ exp_count,
                     double* __restrict__ psum64, int* __restrict__ exp_rows,
                     int* __restrict__ exp_base, int* __restrict__ tile_prefix,
                     int* __restrict__ ready, float* __restrict__ aux_loss, WsHeader* hdr,
                     int nblk, int N, int T, int C_eff, int tile_rows,
                     uint8_t* __restrict__ record, int record_psum_offset,
                     const int* __restrict__ blk_count1, int* __restrict__ exp_count1,
                     SplitPlan split) {
  __shared__ int wc[kScanWarps][32];
  __shared__ double wp[kScanWarps][32];
  __shared__ int is_last;
  pdl_trigger();
  pdl_wait();   // block statistics come from the router
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 32 + lane;
  const int per = (nblk + kScanWarps - 1) / kScanWarps;
  const int b0 = warp * per, b1 = min(nblk, b0 + per);

  // pass 1: this warp's share of blocks, per expert (lane); the counts of up to
  // kRegBlocks blocks stay in registers for pass 2, loads issued before use
  constexpr int kRegBlocks = 16;
  int creg[kRegBlocks];
  int csum = 0;
  double psum = 0.0;
  if (e < N) {
    for (int bb = b0; bb < b1; bb += kRegBlocks) {
      float preg[kRegBlocks];
#pragma unroll
      for (int j = 0; j < kRegBlocks; ++j) {
        const int b = bb + j;
        creg[j] = b < b1 ? blk_count[(size_t)b * N + e] : 0;
        preg[j] = b < b1 ? blk_psum[(size_t)b * N + e] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < kRegBlocks; ++j) {
        csum += creg[j];
        psum += (double)preg[j];
      }
    }
  }
  // top-2: first choices alone, for the aux loss's f
  int c1sum = 0;
  if (blk_count1 != nullptr && e < N)
    for (int b = b0; b < b1; ++b) c1sum += blk_count1[(size_t)b * N + e];
  __shared__ int wc1[kScanWarps][32];
  wc1[warp][lane] = c1sum;
  wc[warp][lane] = csum;
  wp[warp][lane] = psum;
  __syncthreads();
  // pass 2: exclusive offsets in token order
  if (e < N) {
    int off = 0;
    for (int w = 0; w < warp; ++w) off += wc[w][lane];
    if (b1 - b0 <= kRegBlocks) {
#pragma unroll
      for (int j = 0; j < kRegBlocks; ++j) {
        const int b = b0 + j;
        if (b < b1) {
          blk_off[(size_t)b * N + e] = off;
          off += creg[j];
        }
      }
    } else {
      for (int b = b0; b < b1; ++b) {
        const size_t i = (size_t)b * N + e;
        const int c = blk_count[i];
        blk_off[i] = off;
        off += c;
      }
    }
    if (warp == 0) {
      int tot = 0;
      double ps = 0.0;
      for (int w = 0; w < kScanWarps; ++w) { tot += wc[w][lane]; ps += wp[w][lane]; }
      exp_count[e] = tot;
      psum64[e] = ps;
      if (exp_count1 != nullptr) {
        int t1 = 0;
        for (int w = 0; w < kScanWarps; ++w) t1 += wc1[w][lane];
        exp_count1[e] = t1;
      }
      if (record != nullptr) {
        reinterpret_cast<int*>(record)[e] = tot;
        reinterpret_cast<double*>(record + record_psum_offset)[e] = ps;
      }
    }
  }
  if (record != nullptr) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int ticket = atomicAdd(&hdr->done, 1u);
    is_last = (ticket == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // ---- last CTA: scan over experts, tile prefix, aux loss
  __shared__ int s_warp[kScanWarps];
  __shared__ int s_tot_rows, s_tot_tiles;
  __shared__ double s_aux[kScanWarps];
  const int chunk = (N + kScanThreads - 1) / kScanThreads;
  const int e0 = threadIdx.x * chunk, e1 = min(N, e0 + chunk);
  int rows = 0, tiles = 0;
  double aux = 0.0;
  for (int i = e0; i < e1; ++i) {
    const int c = __ldcg(exp_count + i);
    const int m = min(c, C_eff);
    rows += m;
    tiles += (m + tile_rows - 1) / tile_rows;
    const int cf = exp_count1 != nullptr ? __ldcg(exp_count1 + i) : c;   // argmax counts
    aux += (double)cf * __ldcg(psum64 + i);
  }
  int base_rows = block_excl_scan(rows, s_warp, &s_tot_rows);
  int base_tiles = block_excl_scan(tiles, s_warp, &s_tot_tiles);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) aux += __shfl_xor_sync(0xffffffffu, aux, off);
  if (lane == 0) s_aux[warp] = aux;
  __syncthreads();
  // per-call state of the expert FFN kernel: token-tile readiness and work counter
  for (int i = threadIdx.x; i < s_tot_tiles; i += kScanThreads) ready[i] = 0;
  if (threadIdx.x == 0) {
    double a = 0.0;
    for (int w = 0; w < kScanWarps; ++w) a += s_aux[w];
    tile_prefix[N] = s_tot_tiles;
    hdr->next_tile = 0u;
    hdr->gather_prefetch = 2 * s_tot_rows >= T ? 1 : 0;
    // aux = N * sum_i (count_i / T) * (psum_i / T)
    *aux_loss = (float)((double)N * a / ((double)T * (double)T));
    hdr->done = 0u;   // ready for the next call
  }
  for (int i = e0; i < e1; ++i) {
    const int m = min(__ldcg(exp_count + i), C_eff);
    exp_rows[i] = m;
    exp_base[i] = base_rows;
    tile_prefix[i] = base_tiles;
    base_rows += m;
    base_tiles += (m + tile_rows - 1) / tile_rows;
  }
  if (split.factor > 1) {
    // GEMM2 split over K, in expert order while the groups (an expert's
    // 128-feature by token-tile GEMM2 tiles) fit the budget: the split tile
    // prefix, each expert's first group (-1: not split) and the group table
    __shared__ int s_tot_groups, s_tot_tiles2;
    for (int i = threadIdx.x; i < split.max_groups; i += kScanThreads)
      reinterpret_cast<int4*>(split.groups)[i] = make_int4(-1, 0, 0, 0);
    for (int i = threadIdx.x; i < split.max_groups * kSplitFactor; i += kScanThreads)
      split.ready[i] = 0;
    int groups = 0;
    for (int i = e0; i < e1; ++i) {
      const int m = min(__ldcg(exp_count + i), C_eff);
      groups += (m + tile_rows - 1) / tile_rows * split.m_tiles2;
    }
    int g = block_excl_scan(groups, s_warp, &s_tot_groups);
    int tiles2 = 0;
    for (int i = e0; i < e1; ++i) {
      const int m = min(__ldcg(exp_count + i), C_eff);
      const int tl = (m + tile_rows - 1) / tile_rows;
      const int grp = tl * split.m_tiles2;
      const bool on = grp > 0 && g + grp <= split.max_groups;
      tiles2 += tl * (on ? split.factor : 1);
      g += grp;
    }
    int base2 = block_excl_scan(tiles2, s_warp, &s_tot_tiles2);
    g = block_excl_scan(groups, s_warp, &s_tot_groups);   // (its barriers order the -1 fill)
    for (int i = e0; i < e1; ++i) {
      const int m = min(__ldcg(exp_count + i), C_eff);
      const int tl = (m + tile_rows - 1) / tile_rows;
      const int grp = tl * split.m_tiles2;
      const bool on = grp > 0 && g + grp <= split.max_groups;
      split.tile_prefix2[i] = base2;
      split.split_base[i] = on ? g : -1;
      if (on) {
        // group g + mt * tl + nt: m-tile mt of token tile nt (the FFN's numbering)
        for (int mt = 0; mt < split.m_tiles2; ++mt)
          for (int nt = 0; nt < tl; ++nt)
            reinterpret_cast<int4*>(split.groups)[g + mt * tl + nt] = make_int4(i, mt, nt, 0);
      }
      base2 += tl * (on ? split.factor : 1);
      g += grp;
    }
    if (threadIdx.x == 0) split.tile_prefix2[N] = s_tot_tiles2;
  }
}

constexpr int kGatherThreads = 256;
constexpr int kGatherWarps = kGatherThreads / 32;
constexpr int kGatherMaxVecPerLane = 8;   // rows up to 8 x 32 x 16 B = 4 KiB held in registers

// One warp per token.  VEC = bytes per vector move (16 for bf16 rows, 4 for fp32).
// The token's row is loaded before its destination is known (it does not depend
// on the routing), then either stored to its packed expert row or dropped and
// the output row zeroed.
template <int VEC>
__global__ void __launch_bounds__(kGatherThreads)
dispatch_gather_kernel(const uint8_t* __restrict__ x, const int* __restrict__ expert_idx,
                       int* __restrict__ pos_in_expert, const int* __restrict__ blk_off,
                       const int* __restrict__ exp_base, const int* __restrict__ exp_off,
                       int* __restrict__ slot_token, uint8_t* __restrict__ xbuf,
                       uint8_t* __restrict__ out, int T, int N, int C_eff, int row_bytes,
                       int tpb, int prefetch, int kk, WsHeader* hdr) {
  using V = typename std::conditional<VEC == 16, uint4, uint32_t>::type;
  pdl_trigger();
  pdl_wait();   // offsets come from the scan
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // one warp per assignment a = kk t + k (kk = 1: per token; top-2: kk = 2, and a
  // dropped assignment writes nothing: the combine kernel sums the kept ones)
  const int a = blockIdx.x * kGatherWarps + warp;
  if (a >= T * kk) return;
  const int t = a / kk;
  const int nv = row_bytes / VEC;
  const V* src = reinterpret_cast<const V*>(x + (size_t)t * row_bytes);
  V reg[kGatherMaxVecPerLane];
  // prefetch: the row is requested before its destination is known (1: x is
  // still in L2 after the router; 2: when the scan found at least half of the
  // tokens kept, so the few dropped rows read for nothing cost less than the
  // round trip saved); otherwise only kept tokens' rows are read
  const bool in_regs = (prefetch == 1 || (prefetch == 2 && hdr->gather_prefetch != 0)) &&
                       nv <= 32 * kGatherMaxVecPerLane;
  if (in_regs) {
#pragma unroll
    for (int j = 0; j < kGatherMaxVecPerLane; ++j)
      if (lane + 32 * j < nv) reg[j] = src[lane + 32 * j];
  }
  const int e = expert_idx[a];
  const int rank = pos_in_expert[a];            // holds the in-block rank
  if (e < 0 || e >= N) {          // cannot happen: the router clamps its choice
    if (lane == 0) atomicExch(&hdr->err, kDevIndexOutOfRange);
    return;
  }
  const int b = t / tpb;
  // a shard of a global batch: the tokens of earlier ranks come first
  const int off = exp_off != nullptr ? exp_off[e] : 0;
  const int pos = off + blk_off[(size_t)b * N + e] + rank;
  const int base = exp_base[e];
  __syncwarp();
  if (lane == 0) pos_in_expert[a] = pos;
  if (pos < C_eff) {
    const int row = base + pos - off;
    if (!checked_index(row >= 0 && row < T * kk, &hdr->err)) return;
    if (lane == 0) slot_token[row] = a;
    V* dst = reinterpret_cast<V*>(xbuf + (size_t)row * row_bytes);
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < kGatherMaxVecPerLane; ++j)
        if (lane + 32 * j < nv) dst[lane + 32 * j] = reg[j];
    } else {
      for (int i = lane; i < nv; i += 32) dst[i] = src[i];
    }
  } else if (kk == 1 && out != nullptr) {   // (expert parallel: the combine writes zeros)
    V* dst = reinterpret_cast<V*>(out + (size_t)t * row_bytes);
    V z;
    memset(&z, 0, sizeof(V));
    for (int i = lane; i < nv; i += 32) dst[i] = z;
  }
}

// Top-2 combine: out[t] = sum over k of (assignment 2t+k kept ? ybuf[2t+k] : 0),
// the gated rows the GEMM2 epilogue wrote, added in fp32 in choice order and
// rounded once to the activation dtype (a dropped assignment contributes 0; a
// token with both dropped gets a zero row).  One warp per token.
template <typename TA>
__global__ void __launch_bounds__(kGatherThreads)
combine_top2_kernel(const TA* __restrict__ ybuf, const int* __restrict__ pos_in_expert,
                    TA* __restrict__ out, int T, int d, int C_cmp) {
  pdl_trigger();
  pdl_wait();   // rows come from the expert FFN
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kGatherWarps + warp;
  if (t >= T) return;
  const bool k0 = pos_in_expert[2 * t] < C_cmp, k1 = pos_in_expert[2 * t + 1] < C_cmp;
  const TA* y0 = ybuf + (size_t)(2 * t) * d;
  const TA* y1 = y0 + d;
  TA* o = out + (size_t)t * d;
  for (int j = lane; j < d; j += 32) {
    float v = 0.f;
    if (k0) v += static_cast<float>(y0[j]);
    if (k1) v += static_cast<float>(y1[j]);
    o[j] = static_cast<TA>(v);
  }
}

constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedMaxN = 128;
constexpr int kFusedRegVec = 8;   // row vectors per lane held in registers (4 KiB rows at 16 B)

// Scan and gather in one launch (N <= 128): CTA b owns router block b (tpb
// tokens).  Every CTA sums the per-block counts itself - the expert totals and
// the prefix over the blocks before b - so no CTA waits for another; CTA 0 also
// writes the expert bases, the GEMM tile prefix, the aux loss and the expert
// FFN's per-call counters.  Then one warp per token: pos = prefix + in-block
// rank; a kept token records its packed row and is copied there, a dropped
// token's output row is zeroed.  Integer sums are exact in any order; the fp64
// sums of p run in a fixed order (deterministic).
template <int VEC>
__global__ void __launch_bounds__(kFusedThreads)
dispatch_fused_kernel(const uint8_t* __restrict__ x, const int* __restrict__ expert_idx,
                      int* __restrict__ pos_in_expert, const int* __restrict__ blk_count,
                      const float* __restrict__ blk_psum, int* __restrict__ exp_rows,
                      int* __restrict__ exp_base, int* __restrict__ tile_prefix,
                      int* __restrict__ slot_token, int* __restrict__ ready,
                      uint8_t* __restrict__ xbuf, uint8_t* __restrict__ out,
                      float* __restrict__ aux_loss, WsHeader* hdr, int T, int N, int nblk,
                      int tpb, int C_eff, int tile_rows, int row_bytes, int copy_rows) {
  using V = typename std::conditional<VEC == 16, uint4, uint32_t>::type;
  __shared__ int s_tot[kFusedMaxN], s_pre[kFusedMaxN], s_base[kFusedMaxN];
  __shared__ double s_ps[kFusedThreads];
  __shared__ double s_term[kFusedMaxN];
  __shared__ int s_tiles;
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x;
  const int t0 = b * tpb;
  const int ntok = min(tpb, T - t0);
  const int nv = row_bytes / VEC;
  const bool in_regs = copy_rows && nv <= 32 * kFusedRegVec;
  // this warp's first token row: x is a layer input, readable before the wait
  V cur[kFusedRegVec];
  auto load_row = [&](int t, V (&r)[kFusedRegVec]) {
    const V* src = reinterpret_cast<const V*>(x + (size_t)t * row_bytes);
#pragma unroll
    for (int j = 0; j < kFusedRegVec; ++j)
      if (lane + 32 * j < nv) r[j] = src[lane + 32 * j];
  };
  if (in_regs && warp < ntok) load_row(t0 + warp, cur);
  pdl_wait();   // block statistics and ranks come from the router

  for (int e = tid; e < N; e += kFusedThreads) {
    s_tot[e] = 0;
    s_pre[e] = 0;
  }
  // this warp's tokens (i = warp + 16 j): expert and in-block rank, lane j holds
  // token j's, all requested now
  const int my_i = warp + kFusedWarps * lane;
  const int my_e = my_i < ntok ? expert_idx[t0 + my_i] : 0;
  const int my_rank = my_i < ntok ? pos_in_expert[t0 + my_i] : 0;
  __syncthreads();
  // per expert: total over all blocks and prefix over blocks < b (G threads
  // each); the counts are requested in batches of kBatch before they are summed
  const int G = kFusedThreads / N;
  const int ee = tid % N, g = tid / N;
  double ps = 0.0;
  if (g < G) {
    constexpr int kBatch = 16;
    int tot = 0, pre = 0;
    for (int bb0 = g; bb0 < nblk; bb0 += kBatch * G) {
      int c[kBatch];
      float q[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int bb = bb0 + u * G;
        c[u] = bb < nblk ? blk_count[(size_t)bb * N + ee] : 0;
        q[u] = (b == 0 && bb < nblk) ? blk_psum[(size_t)bb * N + ee] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        tot += c[u];
        pre += (bb0 + u * G < b) ? c[u] : 0;
        ps += (double)q[u];
      }
    }
    atomicAdd(&s_tot[ee], tot);
    atomicAdd(&s_pre[ee], pre);
  }
  if (b == 0) s_ps[tid] = ps;
  __syncthreads();
  // packed row bases (and, in CTA 0, the expert FFN's tile prefix): one warp
  if (warp == 0) {
    constexpr int EPL = kFusedMaxN / 32;
    int rows[EPL], tiles[EPL];
    int rs = 0, ts = 0;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane * EPL + j;
      rows[j] = e < N ? min(s_tot[e], C_eff) : 0;
      tiles[j] = (rows[j] + tile_rows - 1) / tile_rows;
      rs += rows[j];
      ts += tiles[j];
    }
    const int rs_in = warp_incl_scan(rs, lane), ts_in = warp_incl_scan(ts, lane);
    int run = rs_in - rs, trun = ts_in - ts;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane * EPL + j;
      if (e < N) {
        s_base[e] = run;
        if (b == 0) {
          exp_rows[e] = rows[j];
          exp_base[e] = run;
          tile_prefix[e] = trun;
        }
      }
      run += rows[j];
      trun += tiles[j];
    }
    const int total_tiles = __shfl_sync(0xffffffffu, ts_in, 31);
    if (lane == 0) {
      s_tiles = total_tiles;
      if (b == 0) tile_prefix[N] = total_tiles;
    }
  }
  __syncthreads();
  if (b == 0) {
    // per-call state of the expert FFN kernel: token-tile readiness, work counter
    for (int i = tid; i < s_tiles; i += kFusedThreads) ready[i] = 0;
    // aux = N * sum_i (count_i / T) * (sum_t p_t,i / T); sums in a fixed order
    if (tid < N) {
      double P = 0.0;
      for (int g2 = 0; g2 < G; ++g2) P += s_ps[g2 * N + tid];
      s_term[tid] = (double)s_tot[tid] * P;
    }
    __syncthreads();
    if (tid == 0) {
      double a = 0.0;
      for (int e = 0; e < N; ++e) a += s_term[e];
      *aux_loss = (float)((double)N * a / ((double)T * (double)T));
      hdr->next_tile = 0u;
    }
  }
  // one warp per token; the next token's row is requested before this one's
  // destination is known
  for (int i = warp, j = 0; i < ntok; i += kFusedWarps, ++j) {
    const int t = t0 + i;
    V nxt[kFusedRegVec];
    const bool more = i + kFusedWarps < ntok;
    if (in_regs && more) load_row(t + kFusedWarps, nxt);
    const int e = __shfl_sync(0xffffffffu, my_e, j);
    if (e < 0 || e >= N) {        // cannot happen: the router clamps its choice
      if (lane == 0) atomicExch(&hdr->err, kDevIndexOutOfRange);
      return;
    }
    const int pos = s_pre[e] + __shfl_sync(0xffffffffu, my_rank, j);   // prefix + in-block rank
    __syncwarp();
    if (lane == 0) pos_in_expert[t] = pos;
    if (pos < C_eff) {
      const int row = s_base[e] + pos;
      if (!checked_index(row >= 0 && row < T, &hdr->err)) return;
      if (lane == 0) slot_token[row] = t;
      if (copy_rows) {
        V* dst = reinterpret_cast<V*>(xbuf + (size_t)row * row_bytes);
        if (in_regs) {
#pragma unroll
          for (int j = 0; j < kFusedRegVec; ++j)
            if (lane + 32 * j < nv) dst[lane + 32 * j] = cur[j];
        } else {
          const V* src = reinterpret_cast<const V*>(x + (size_t)t * row_bytes);
          for (int j = lane; j < nv; j += 32) dst[j] = src[j];
        }
      }
    } else {
      V* dst = reinterpret_cast<V*>(out + (size_t)t * row_bytes);
      V z;
      memset(&z, 0, sizeof(V));
      for (int j = lane; j < nv; j += 32) dst[j] = z;
    }
    if (in_regs && more) {
#pragma unroll
      for (int j = 0; j < kFusedRegVec; ++j) cur[j] = nxt[j];
    }
  }
}

constexpr int kCombineThreads = 512;
constexpr int kCombineWarps = kCombineThreads / 32;

// A global batch sharded over `world` ranks by contiguous token ranges, rank
// order = token order.  From every rank's exchange record (expert totals of its
// tokens and their sums of p), one CTA computes for this rank:
//   exp_off[e]   tokens of expert e on earlier ranks, so that a local token's
//                position is exp_off[e] + its position among this rank's tokens
//                (the cumulative sum over the expert's column in global token
//                order, "The routing mechanics in detail");
//   exp_rows[e]  this rank's kept tokens of e: those whose global position is
//                below C, min(count, max(0, C - exp_off[e]));
//   packed bases, the GEMM tile prefix and the FFN's per-call state;
//   the aux loss N * sum_i f_i P_i over the whole batch, with each expert's
//   totals summed in rank order (every rank computes the same value).
// C_cap = min(C, T_total).  A record set whose counts do not add up to
// T_total (ranks disagreeing on the batch) or to this rank's T raises
// kDevIndexOutOfRange; the rows are then clamped to stay in range.
__global__ void __launch_bounds__(kCombineThreads)
shard_combine_kernel(const uint8_t* __restrict__ gathered, int record_bytes,
                     int record_psum_offset, int rank, int world, int N, int T_local,
                     int T_total, int C_cap, int tile_rows,
                     const int* __restrict__ exp_count, int* __restrict__ exp_off,
                     int* __restrict__ exp_rows, int* __restrict__ exp_base,
                     int* __restrict__ tile_prefix, int* __restrict__ ready,
                     float* __restrict__ aux_loss, WsHeader* hdr) {
  __shared__ int s_warp[kCombineWarps];
  __shared__ int s_tot_rows, s_tot_tiles;
  __shared__ double s_aux[kCombineWarps];
  __shared__ long long s_cnt[2][kCombineWarps];
  pdl_trigger();
  pdl_wait();   // the records were gathered after the local scan
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = (N + kCombineThreads - 1) / kCombineThreads;
  const int e0 = threadIdx.x * chunk, e1 = min(N, e0 + chunk);
  int rows = 0, tiles = 0;
  long long all_tok = 0, my_tok = 0;
  double aux = 0.0;
  bool consistent = true;
  for (int i = e0; i < e1; ++i) {
    long long before = 0, tot = 0;
    int mine = 0;
    double ps = 0.0;
    for (int g = 0; g < world; ++g) {
      const uint8_t* rec = gathered + static_cast<size_t>(g) * record_bytes;
      const int c = reinterpret_cast<const int*>(rec)[i];
      tot += c;
      if (g < rank) before += c;
      if (g == rank) mine = c;
      ps += reinterpret_cast<const double*>(rec + record_psum_offset)[i];
    }
    // this rank's own count comes from its scan (the record should repeat it):
    // the kept rows then never exceed the rows this rank holds
    const int own = exp_count != nullptr ? exp_count[i] : 0;   // null: no local tokens
    consistent = consistent && own == mine && before >= 0 && before <= T_total;
    const long long room = static_cast<long long>(C_cap) - before;
    const int m = static_cast<int>(max(0ll, min(static_cast<long long>(own), room)));
    rows += m;
    tiles += (m + tile_rows - 1) / tile_rows;
    aux += static_cast<double>(tot) * ps;
    all_tok += tot;
    my_tok += own;
    exp_off[i] = static_cast<int>(min(max(before, 0ll), static_cast<long long>(T_total)));
    exp_rows[i] = m;
  }
  if (!consistent) atomicExch(&hdr->err, kDevIndexOutOfRange);
  int base_rows = block_excl_scan(rows, s_warp, &s_tot_rows);
  int base_tiles = block_excl_scan(tiles, s_warp, &s_tot_tiles);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    aux += __shfl_xor_sync(0xffffffffu, aux, off);
    all_tok += __shfl_xor_sync(0xffffffffu, all_tok, off);
    my_tok += __shfl_xor_sync(0xffffffffu, my_tok, off);
  }
  if (lane == 0) {
    s_aux[warp] = aux;
    s_cnt[0][warp] = all_tok;
    s_cnt[1][warp] = my_tok;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < s_tot_tiles; i += kCombineThreads) ready[i] = 0;
  if (threadIdx.x == 0) {
    double a = 0.0;
    long long at = 0, mt = 0;
    for (int w = 0; w < kCombineWarps; ++w) {
      a += s_aux[w];
      at += s_cnt[0][w];
      mt += s_cnt[1][w];
    }
    if (at != T_total || mt != T_local) atomicExch(&hdr->err, kDevIndexOutOfRange);
    checked_index(s_tot_rows <= T_local, &hdr->err);
    tile_prefix[N] = s_tot_tiles;
    hdr->next_tile = 0u;
    *aux_loss = (float)((double)N * a / ((double)T_total * (double)T_total));
  }
  for (int i = e0; i < e1; ++i) {
    const int m = exp_rows[i];
    exp_base[i] = base_rows;
    tile_prefix[i] = base_tiles;
    base_rows += m;
    base_tiles += (m + tile_rows - 1) / tile_rows;
  }
}

// ------------------------------------------------------------------ expert parallel
// Experts are split over `world` ranks, rank r owning experts [r L, r L + L)
// (L = N / world); the tokens of one global batch are split by contiguous
// ranges as in shard_combine_kernel.  From the gathered exchange records every
// rank knows, for every rank g and expert e, how many of g's tokens of e are
// kept: m[g][e] = min(count[g][e], max(0, C - offset[g][e])), the kept global
// positions of e being [offset[g][e], offset[g][e] + m[g][e]).  Rank g sends
// its kept rows packed by expert (its own packed buffer), so the rows for owner
// r form one contiguous segment; the owner receives, source by source, blocks
// (g, local expert l) of m[g][e] rows, and ep_plan_kernel lays out where each
// block goes in the owner's per-expert packed buffer: expert e's rows in global
// position order (source rank, then token order), exactly the rows and order
// of the unsharded layer.
__global__ void __launch_bounds__(kCombineThreads)
ep_plan_kernel(const uint8_t* __restrict__ gathered, int record_bytes, int record_psum_offset,
               int rank, int world, int L, int C_cap, int tile_rows, int* __restrict__ blk_src,
               int* __restrict__ blk_dst, int* __restrict__ blk_n, int* __restrict__ ep_rows,
               int* __restrict__ ep_base, int* __restrict__ ep_tile_prefix,
               int* __restrict__ ready, int max_rows, WsHeader* hdr) {
  __shared__ int s_warp[kCombineWarps];
  __shared__ int s_tot_rows, s_tot_tiles, s_seg_total;
  pdl_trigger();
  pdl_wait();
  const int chunk = (L + kCombineThreads - 1) / kCombineThreads;
  const int l0 = threadIdx.x * chunk, l1 = min(L, l0 + chunk);
  // per local expert: the kept rows of every source (their positions tile
  // [0, K_e) in source order)
  int rows = 0, tiles = 0;
  for (int l = l0; l < l1; ++l) {
    const int e = rank * L + l;
    long long before = 0;
    int kept = 0;
    for (int g = 0; g < world; ++g) {
      const int c = reinterpret_cast<const int*>(gathered + static_cast<size_t>(g) * record_bytes)[e];
      const long long room = static_cast<long long>(C_cap) - before;
      const int m = static_cast<int>(max(0ll, min(static_cast<long long>(c), room)));
      blk_n[g * L + l] = m;
      blk_dst[g * L + l] = static_cast<int>(min(before, static_cast<long long>(C_cap)));
      before += c;
      kept += m;
    }
    ep_rows[l] = kept;
    rows += kept;
    tiles += (kept + tile_rows - 1) / tile_rows;
  }
  int base_rows = block_excl_scan(rows, s_warp, &s_tot_rows);
  int base_tiles = block_excl_scan(tiles, s_warp, &s_tot_tiles);
  for (int l = l0; l < l1; ++l) {
    ep_base[l] = base_rows;
    ep_tile_prefix[l] = base_tiles;
    for (int g = 0; g < world; ++g) blk_dst[g * L + l] += base_rows;
    base_rows += ep_rows[l];
    base_tiles += (ep_rows[l] + tile_rows - 1) / tile_rows;
  }
  // receive order: source g, then local expert l; blk_src = exclusive prefix
  int seg_base = 0;
  for (int g = 0; g < world; ++g) {
    int part = 0;
    for (int l = l0; l < l1; ++l) part += blk_n[g * L + l];
    int off = block_excl_scan(part, s_warp, &s_seg_total) + seg_base;
    for (int l = l0; l < l1; ++l) {
      blk_src[g * L + l] = off;
      off += blk_n[g * L + l];
    }
    seg_base += s_seg_total;
    __syncthreads();
  }
  if (s_tot_rows > max_rows) atomicExch(&hdr->err, kDevIndexOutOfRange);   // cannot happen
  for (int i = threadIdx.x; i < s_tot_tiles; i += kCombineThreads) ready[i] = 0;
  if (threadIdx.x == 0) {
    ep_tile_prefix[L] = s_tot_tiles;
    hdr->next_tile = 0u;
  }
}

// Moves rows between the receive order (source rank, local expert) and the
// owner's per-expert packed buffer: dir 0 copies recv[i] to packed[dst], dir 1
// copies packed[dst] back to recv[i] (the return trip).  One warp per row i of
// the receive order; its block is the last entry whose start is <= i.
template <int VEC>
__global__ void __launch_bounds__(kGatherThreads)
ep_permute_kernel(uint8_t* __restrict__ recv, uint8_t* __restrict__ packed,
                  const int* __restrict__ blk_src, const int* __restrict__ blk_dst,
                  const int* __restrict__ blk_n, int nblocks, int n_recv, int max_rows,
                  int row_bytes, int dir, WsHeader* hdr) {
  using V = typename std::conditional<VEC == 16, uint4, uint32_t>::type;
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kGatherWarps + warp;
  const int total = blk_src[nblocks - 1] + blk_n[nblocks - 1];
  if (i >= total) return;
  if (i >= n_recv) {              // more rows than the caller's receive buffer holds
    if (lane == 0) atomicExch(&hdr->err, kDevIndexOutOfRange);
    return;
  }
  int lo = 0, hi = nblocks;       // last j with blk_src[j] <= i
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (blk_src[mid] <= i) lo = mid; else hi = mid;
  }
  const int row = blk_dst[lo] + (i - blk_src[lo]);
  if (row < 0 || row >= max_rows) {
    if (lane == 0) atomicExch(&hdr->err, kDevIndexOutOfRange);
    return;
  }
  const int nv = row_bytes / VEC;
  V* r = reinterpret_cast<V*>(recv + static_cast<size_t>(i) * row_bytes);
  V* p = reinterpret_cast<V*>(packed + static_cast<size_t>(row) * row_bytes);
  if (dir == 0) {
    for (int j = lane; j < nv; j += 32) p[j] = r[j];
  } else {
    for (int j = lane; j < nv; j += 32) r[j] = p[j];
  }
}

// Source side of the return trip: the rows came back in this rank's packed
// order (expert, then token order): out[t] = g_t * row for a kept token, zero
// for a dropped one.  One warp per token.
template <typename TA>
__global__ void __launch_bounds__(kGatherThreads)
ep_combine_kernel(const TA* __restrict__ ret, const int* __restrict__ expert_idx,
                  const float* __restrict__ gate, const int* __restrict__ pos_in_expert,
                  const int* __restrict__ exp_base, const int* __restrict__ exp_off,
                  TA* __restrict__ out, int T, int d, int C_cmp, WsHeader* hdr) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kGatherWarps + warp;
  if (t >= T) return;
  const int e = expert_idx[t], pos = pos_in_expert[t];
  TA* o = out + static_cast<size_t>(t) * d;
  if (pos < C_cmp) {
    const int row = exp_base[e] + pos - exp_off[e];
    if (row < 0 || row >= T) {
      if (lane == 0) atomicExch(&hdr->err, kDevIndexOutOfRange);
      return;
    }
    const float g = gate[t];
    const TA* y = ret + static_cast<size_t>(row) * d;
    for (int j = lane; j < d; j += 32) o[j] = static_cast<TA>(g * static_cast<float>(y[j]));
  } else {
    for (int j = lane; j < d; j += 32) o[j] = static_cast<TA>(0.f);
  }
}

// ---------------------------------------------------------------- No-Token-Left-Behind
// Two stages (paper-graph summary of arXiv 2101.03961, Appendix B: tokens that
// overflow their first expert go to their second choice).  Stage 1 is the top-1
// dispatch of the first choices (the scan over the router's first-choice block
// counts gives each block's offsets); stage 2 ranks, in token order, the tokens
// stage 1 dropped among those with the same second choice, and a second scan
// gives the blocks' offsets; a token rerouted to expert e takes position
// min(first-choice count of e, C) + its stage-2 offset and rank.
constexpr int kNtlbThreads = 256;

// Stage 2 for one token block: each token's stage-1 position (written to
// pos_in_expert[2t]); the block's overflow tokens' in-block ranks per second
// choice (rank2) and counts (blk_cnt2 row b, every expert).
__global__ void __launch_bounds__(kNtlbThreads)
ntlb_stage2_kernel(const int* __restrict__ expert_idx, const int* __restrict__ blk_off1,
                   int* __restrict__ pos_in_expert, int* __restrict__ rank2,
                   int* __restrict__ blk_cnt2, int T, int N, int tpb, int C_cmp, int* err) {
  __shared__ int e1s[kTokensPerBlock], e2s[kTokensPerBlock], over[kTokensPerBlock];
  pdl_trigger();
  pdl_wait();   // the first-choice offsets come from the stage-1 scan
  const int b = blockIdx.x, t0 = b * tpb, nt = min(tpb, T - t0);
  int* cnt_row = blk_cnt2 + static_cast<size_t>(b) * N;
  for (int n = threadIdx.x; n < N; n += kNtlbThreads) cnt_row[n] = 0;
  for (int i = threadIdx.x; i < nt; i += kNtlbThreads) {
    int e1 = expert_idx[2 * (t0 + i)], e2 = expert_idx[2 * (t0 + i) + 1];
    if (!checked_index(e1 >= 0 && e1 < N && e2 >= 0 && e2 < N, err)) e1 = e2 = 0;
    e1s[i] = e1;
    e2s[i] = e2;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nt; i += kNtlbThreads) {
    const int e = e1s[i];
    int r = 0;
    for (int j = 0; j < i; ++j) r += (e1s[j] == e);
    const int p1 = blk_off1[static_cast<size_t>(b) * N + e] + r;
    pos_in_expert[2 * (t0 + i)] = p1;
    over[i] = p1 >= C_cmp ? 1 : 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nt; i += kNtlbThreads) {
    if (!over[i]) continue;
    const int e = e2s[i];
    int r = 0;
    for (int j = 0; j < i; ++j) r += over[j] & (e2s[j] == e);
    rank2[t0 + i] = r;
    if (r == 0) {   // the block's first overflow token with this second choice counts them
      int c = 1;
      for (int j = i + 1; j < nt; ++j) c += over[j] & (e2s[j] == e);
      cnt_row[e] = c;
    }
  }
}

// Expert level (one CTA): kept rows per expert (stage-1 rows, then the stage-2
// rows up to the capacity), packed-row bases, tile prefix, the FFN's per-call
// state, and the aux loss from the first-choice counts.
__global__ void __launch_bounds__(kScanThreads)
ntlb_finish_kernel(const int* __restrict__ tot1, const int* __restrict__ tot2,
                   const double* __restrict__ psum64, int* __restrict__ exp_rows,
                   int* __restrict__ exp_base, int* __restrict__ tile_prefix,
                   int* __restrict__ ready, float* __restrict__ aux_loss, WsHeader* hdr, int N,
                   int T, int C_cmp, int tile_rows) {
  __shared__ int s_warp[kScanWarps];
  __shared__ int s_tot_rows, s_tot_tiles;
  __shared__ double s_aux[kScanWarps];
  pdl_trigger();
  pdl_wait();   // the stage-2 totals come from the second scan
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = (N + kScanThreads - 1) / kScanThreads;
  const int e0 = threadIdx.x * chunk, e1 = min(N, e0 + chunk);
  auto rows_of = [&](int i) {
    const int k1 = min(tot1[i], C_cmp);
    return k1 + min(tot2[i], C_cmp - k1);
  };
  int rows = 0, tiles = 0;
  double aux = 0.0;
  for (int i = e0; i < e1; ++i) {
    const int m = rows_of(i);
    rows += m;
    tiles += (m + tile_rows - 1) / tile_rows;
    aux += static_cast<double>(tot1[i]) * psum64[i];
  }
  int base_rows = block_excl_scan(rows, s_warp, &s_tot_rows);
  int base_tiles = block_excl_scan(tiles, s_warp, &s_tot_tiles);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) aux += __shfl_xor_sync(0xffffffffu, aux, off);
  if (lane == 0) s_aux[warp] = aux;
  __syncthreads();
  for (int i = threadIdx.x; i < s_tot_tiles; i += kScanThreads) ready[i] = 0;
  if (threadIdx.x == 0) {
    double a = 0.0;
    for (int w = 0; w < kScanWarps; ++w) a += s_aux[w];
    tile_prefix[N] = s_tot_tiles;
    hdr->next_tile = 0u;
    *aux_loss = static_cast<float>(static_cast<double>(N) * a /
                                   (static_cast<double>(T) * static_cast<double>(T)));
  }
  for (int i = e0; i < e1; ++i) {
    const int m = rows_of(i);
    exp_rows[i] = m;
    exp_base[i] = base_rows;
    tile_prefix[i] = base_tiles;
    base_rows += m;
    base_tiles += (m + tile_rows - 1) / tile_rows;
  }
}

// One warp per token: the expert that keeps it (the first choice in stage 1,
// else the second in stage 2, else none), its position (pos_in_expert[2t + 1]:
// the stage-2 position, -1 for a token stage 1 kept), the packed row, the row
// of x copied there and the keeping expert's router probability; a token
// neither stage keeps gets a zero output row.
template <int VEC>
__global__ void __launch_bounds__(kGatherThreads)
ntlb_gather_kernel(const uint8_t* __restrict__ x, const int* __restrict__ expert_idx,
                   const float* __restrict__ gate, int* __restrict__ pos_in_expert,
                   const int* __restrict__ rank2, const int* __restrict__ blk_off2,
                   const int* __restrict__ tot1, const int* __restrict__ exp_base,
                   int* __restrict__ slot_token, float* __restrict__ gsel,
                   uint8_t* __restrict__ xbuf, uint8_t* __restrict__ out, int T, int N, int tpb,
                   int C_cmp, int row_bytes, int* err) {
  using V = typename std::conditional<VEC == 16, uint4, uint32_t>::type;
  pdl_trigger();
  pdl_wait();   // bases come from the finish kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kGatherWarps + warp;
  if (t >= T) return;
  int e1 = expert_idx[2 * t], e2 = expert_idx[2 * t + 1];
  if (!checked_index(e1 >= 0 && e1 < N && e2 >= 0 && e2 < N, err)) e1 = e2 = 0;
  const int p1 = pos_in_expert[2 * t];
  int e = -1, pos = 0, p2 = -1;
  float g = 0.f;
  if (p1 < C_cmp) {
    e = e1;
    pos = p1;
    g = gate[2 * t];
  } else {
    const int b = t / tpb;
    p2 = min(tot1[e2], C_cmp) + blk_off2[static_cast<size_t>(b) * N + e2] + rank2[t];
    if (p2 < C_cmp) {
      e = e2;
      pos = p2;
      g = gate[2 * t + 1];
    }
  }
  if (lane == 0) pos_in_expert[2 * t + 1] = p2;
  const int nv = row_bytes / VEC;
  if (e >= 0) {
    const int row = exp_base[e] + pos;
    if (!checked_index(row >= 0 && row < T, err)) return;
    if (lane == 0) {
      slot_token[row] = t;
      gsel[t] = g;
    }
    const V* src = reinterpret_cast<const V*>(x + static_cast<size_t>(t) * row_bytes);
    V* dst = reinterpret_cast<V*>(xbuf + static_cast<size_t>(row) * row_bytes);
    for (int i = lane; i < nv; i += 32) dst[i] = src[i];
  } else {
    V* dst = reinterpret_cast<V*>(out + static_cast<size_t>(t) * row_bytes);
    V z;
    memset(&z, 0, sizeof(V));
    for (int i = lane; i < nv; i += 32) dst[i] = z;
  }
}

}  // namespace

bool dispatch_fused_ok(const Shape& s) {
  const int64_t elem = s.dtype == 1 ? 2 : 4;
  return s.topk == 1 && !s.sharded && s.N <= kFusedMaxN && s.T * s.d * elem <= (int64_t{16} << 20);
}

cudaError_t launch_dispatch_fused(const Shape& s, const Workspace& ws, const void* x,
                                  const int* expert_idx, int* pos_in_expert, void* out,
                                  float* aux_loss, cudaStream_t stream) {
  const int elem = s.dtype == 1 ? 2 : 4;
  const int row_bytes = (int)(s.d * elem);
  const bool vec16 = (row_bytes % 16 == 0) && ((reinterpret_cast<uintptr_t>(x) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(out) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(ws.xbuf) & 15) == 0);
  const cudaError_t e = launch_dependent(
      vec16 ? dispatch_fused_kernel<16> : dispatch_fused_kernel<4>, dim3(s.nblk),
      dim3(kFusedThreads), 0, stream, static_cast<const uint8_t*>(x), expert_idx, pos_in_expert,
      static_cast<const int*>(ws.blk_count), static_cast<const float*>(ws.blk_psum), ws.exp_rows,
      ws.exp_base, ws.tile_prefix, ws.slot_token, ws.ready, static_cast<uint8_t*>(ws.xbuf),
      static_cast<uint8_t*>(out), aux_loss, ws.hdr, (int)s.T, (int)s.N, s.nblk, s.tpb,
      (int)s.C_eff, s.tile_rows, row_bytes, 1);
  count_launch();
  return e;
}

cudaError_t launch_dispatch_scan(const Shape& s, const Workspace& ws, float* aux_loss,
                                 void* record, cudaStream_t stream) {
  const int grid = (int)((s.N + 31) / 32);
  const cudaError_t e = launch_dependent(
      dispatch_scan_kernel, dim3(grid), dim3(kScanThreads), 0, stream, ws.blk_count, ws.blk_psum,
      ws.blk_off, ws.exp_count, ws.psum64, ws.exp_rows, ws.exp_base, ws.tile_prefix, ws.ready,
      aux_loss, ws.hdr, s.nblk, (int)s.N, (int)s.T, (int)s.C_eff, s.tile_rows,
      static_cast<uint8_t*>(record), (int)shard_record_psum_offset(s.N),
      static_cast<const int*>(s.topk == 2 ? ws.blk_count1 : nullptr),
      s.topk == 2 ? ws.exp_count1 : nullptr,
      SplitPlan{s.ffn_split, (int)((s.d + 127) / 128), kSplitMaxGroups, ws.tile_prefix2,
                ws.split_base, ws.split_grp, ws.split_ready});
  count_launch();
  return e;
}

size_t shard_record_psum_offset(int64_t N) {
  return (static_cast<size_t>(N) * 4 + 15) / 16 * 16;
}

size_t shard_record_bytes(int64_t N) {   // a multiple of 16, so records can sit back to back
  return (shard_record_psum_offset(N) + static_cast<size_t>(N) * 8 + 15) / 16 * 16;
}

cudaError_t launch_shard_combine(const Shape& s, const Workspace& ws, const void* gathered,
                                 int rank, int world, float* aux_loss, cudaStream_t stream) {
  const cudaError_t e = launch_dependent(
      shard_combine_kernel, dim3(1), dim3(kCombineThreads), 0, stream,
      static_cast<const uint8_t*>(gathered), (int)shard_record_bytes(s.N),
      (int)shard_record_psum_offset(s.N), rank, world, (int)s.N, (int)s.T, (int)s.T_total,
      (int)s.C_cmp, s.tile_rows, s.T > 0 ? static_cast<const int*>(ws.exp_count) : nullptr,
      ws.exp_off, ws.exp_rows,
      ws.exp_base, ws.tile_prefix, ws.ready, aux_loss, ws.hdr);
  count_launch();
  return e;
}

cudaError_t launch_dispatch_gather(const Shape& s, const Workspace& ws, const void* x,
                                   const int* expert_idx, int* pos_in_expert, void* out,
                                   cudaStream_t stream) {
  const int grid = (int)((s.T * s.topk + kGatherWarps - 1) / kGatherWarps);
  const int elem = s.dtype == 1 ? 2 : 4;
  const int row_bytes = (int)(s.d * elem);
  const bool vec16 = (row_bytes % 16 == 0) && ((reinterpret_cast<uintptr_t>(x) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(out) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(ws.xbuf) & 15) == 0);
  const cudaError_t e = launch_dependent(
      vec16 ? dispatch_gather_kernel<16> : dispatch_gather_kernel<4>, dim3(grid),
      dim3(kGatherThreads), 0, stream, static_cast<const uint8_t*>(x), expert_idx, pos_in_expert,
      static_cast<const int*>(ws.blk_off), static_cast<const int*>(ws.exp_base),
      static_cast<const int*>(s.sharded ? ws.exp_off : nullptr), ws.slot_token,
      static_cast<uint8_t*>(ws.xbuf), static_cast<uint8_t*>(out), (int)s.T, (int)s.N,
      (int)s.C_cmp, row_bytes, s.tpb,
      s.T * (int64_t)row_bytes <= (int64_t{48} << 20) ? 1 : (s.sharded ? 0 : 2), s.topk, ws.hdr);
  count_launch();
  return e;
}

cudaError_t launch_combine_top2(const Shape& s, const Workspace& ws, const int* pos_in_expert,
                                void* out, cudaStream_t stream) {
  const int grid = (int)((s.T + kGatherWarps - 1) / kGatherWarps);
  cudaError_t e;
  if (s.dtype == 1) {
    e = launch_dependent(combine_top2_kernel<__nv_bfloat16>, dim3(grid), dim3(kGatherThreads), 0,
                         stream, static_cast<const __nv_bfloat16*>(ws.ybuf), pos_in_expert,
                         static_cast<__nv_bfloat16*>(out), (int)s.T, (int)s.d, (int)s.C_cmp);
  } else {
    e = launch_dependent(combine_top2_kernel<float>, dim3(grid), dim3(kGatherThreads), 0,
                         stream, static_cast<const float*>(ws.ybuf), pos_in_expert,
                         static_cast<float*>(out), (int)s.T, (int)s.d, (int)s.C_cmp);
  }
  count_launch();
  return e;
}

cudaError_t launch_ep_plan(const EpPlan& ep, const void* gathered, cudaStream_t stream) {
  const cudaError_t e = launch_dependent(
      ep_plan_kernel, dim3(1), dim3(kCombineThreads), 0, stream,
      static_cast<const uint8_t*>(gathered), (int)shard_record_bytes(ep.N),
      (int)shard_record_psum_offset(ep.N), ep.rank, ep.world, ep.L, (int)ep.C_cmp,
      ep.tile_rows, ep.blk_src, ep.blk_dst, ep.blk_n, ep.rows, ep.base, ep.tile_prefix, ep.ready,
      (int)ep.max_rows, ep.hdr);
  count_launch();
  return e;
}

cudaError_t launch_ep_permute(const EpPlan& ep, void* recv, void* packed, int64_t n_recv,
                              int row_bytes, int dir, cudaStream_t stream) {
  if (n_recv <= 0) return cudaSuccess;
  const int grid = (int)((n_recv + kGatherWarps - 1) / kGatherWarps);
  const bool vec16 = row_bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(recv) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(packed) & 15) == 0;
  const cudaError_t e = launch_dependent(
      vec16 ? ep_permute_kernel<16> : ep_permute_kernel<4>, dim3(grid), dim3(kGatherThreads), 0,
      stream, static_cast<uint8_t*>(recv), static_cast<uint8_t*>(packed),
      static_cast<const int*>(ep.blk_src), static_cast<const int*>(ep.blk_dst),
      static_cast<const int*>(ep.blk_n), ep.world * ep.L, (int)n_recv, (int)ep.max_rows,
      row_bytes, dir, ep.hdr);
  count_launch();
  return e;
}

cudaError_t launch_ep_combine(const Shape& s, const Workspace& ws, const void* ret,
                              const int* expert_idx, const float* gate,
                              const int* pos_in_expert, void* out, cudaStream_t stream) {
  if (s.T <= 0) return cudaSuccess;
  const int grid = (int)((s.T + kGatherWarps - 1) / kGatherWarps);
  cudaError_t e;
  if (s.dtype == 1) {
    e = launch_dependent(ep_combine_kernel<__nv_bfloat16>, dim3(grid), dim3(kGatherThreads), 0,
                         stream, static_cast<const __nv_bfloat16*>(ret), expert_idx, gate,
                         pos_in_expert, static_cast<const int*>(ws.exp_base),
                         static_cast<const int*>(ws.exp_off), static_cast<__nv_bfloat16*>(out),
                         (int)s.T, (int)s.d, (int)s.C_cmp, ws.hdr);
  } else {
    e = launch_dependent(ep_combine_kernel<float>, dim3(grid), dim3(kGatherThreads), 0, stream,
                         static_cast<const float*>(ret), expert_idx, gate, pos_in_expert,
                         static_cast<const int*>(ws.exp_base),
                         static_cast<const int*>(ws.exp_off), static_cast<float*>(out),
                         (int)s.T, (int)s.d, (int)s.C_cmp, ws.hdr);
  }
  count_launch();
  return e;
}


// ---------------------------------------------------------------- No-Token-Left-Behind launches
static cudaError_t launch_scan_totals(const Shape& s, const Workspace& ws, const int* blk_cnt,
                               int* blk_off, int* exp_cnt, cudaStream_t stream) {
  // the scan kernel's shard mode: per-block offsets and per-expert totals only
  // (its expert-level part is left to ntlb_finish_kernel)
  const int grid = (int)((s.N + 31) / 32);
  const cudaError_t e = launch_dependent(
      dispatch_scan_kernel, dim3(grid), dim3(kScanThreads), 0, stream, blk_cnt, ws.blk_psum,
      blk_off, exp_cnt, ws.psum64, ws.exp_rows, ws.exp_base, ws.tile_prefix, ws.ready,
      static_cast<float*>(nullptr), ws.hdr, s.nblk, (int)s.N, (int)s.T, (int)s.C_eff,
      s.tile_rows, static_cast<uint8_t*>(ws.ntlb_rec), (int)shard_record_psum_offset(s.N),
      static_cast<const int*>(nullptr), static_cast<int*>(nullptr),
      SplitPlan{1, 1, 0, nullptr, nullptr, nullptr, nullptr});
  count_launch();
  return e;
}

cudaError_t launch_ntlb_positions(const Shape& s, const Workspace& ws, const int* expert_idx,
                                  int* pos_in_expert, float* aux_loss, cudaStream_t stream) {
  cudaError_t e;
  // stage 1: offsets of the first choices (the router's first-choice block counts)
  if ((e = launch_scan_totals(s, ws, ws.blk_count1, ws.blk_off, ws.exp_count1, stream)) !=
      cudaSuccess)
    return e;
  e = launch_dependent(ntlb_stage2_kernel, dim3(s.nblk), dim3(kNtlbThreads), 0, stream,
                       expert_idx, static_cast<const int*>(ws.blk_off), pos_in_expert,
                       ws.ntlb_rank2, ws.blk_count, (int)s.T, (int)s.N, s.tpb, (int)s.C_cmp,
                       &ws.hdr->err);
  count_launch();
  if (e != cudaSuccess) return e;
  // stage 2: offsets of the overflow tokens per second choice
  if ((e = launch_scan_totals(s, ws, ws.blk_count, ws.blk_off, ws.exp_count, stream)) !=
      cudaSuccess)
    return e;
  e = launch_dependent(ntlb_finish_kernel, dim3(1), dim3(kScanThreads), 0, stream,
                       static_cast<const int*>(ws.exp_count1),
                       static_cast<const int*>(ws.exp_count),
                       static_cast<const double*>(ws.psum64), ws.exp_rows, ws.exp_base,
                       ws.tile_prefix, ws.ready, aux_loss, ws.hdr, (int)s.N, (int)s.T,
                       (int)s.C_cmp, s.tile_rows);
  count_launch();
  return e;
}

cudaError_t launch_ntlb_gather(const Shape& s, const Workspace& ws, const void* x,
                               const int* expert_idx, const float* gate, int* pos_in_expert,
                               void* out, cudaStream_t stream) {
  const int elem = s.dtype == 1 ? 2 : 4;
  const int row_bytes = (int)(s.d * elem);
  const bool vec16 = (row_bytes % 16 == 0) && ((reinterpret_cast<uintptr_t>(x) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(out) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(ws.xbuf) & 15) == 0);
  const int grid = (int)((s.T + kGatherWarps - 1) / kGatherWarps);
  const cudaError_t e = launch_dependent(vec16 ? ntlb_gather_kernel<16> : ntlb_gather_kernel<4>, dim3(grid),
                       dim3(kGatherThreads), 0, stream, static_cast<const uint8_t*>(x),
                       expert_idx, gate, pos_in_expert, static_cast<const int*>(ws.ntlb_rank2),
                       static_cast<const int*>(ws.blk_off),
                       static_cast<const int*>(ws.exp_count1),
                       static_cast<const int*>(ws.exp_base), ws.slot_token, ws.ntlb_gate,
                       static_cast<uint8_t*>(ws.xbuf), static_cast<uint8_t*>(out), (int)s.T,
                       (int)s.N, s.tpb, (int)s.C_cmp, row_bytes, &ws.hdr->err);
  count_launch();
  return e;
}

}  // namespace swl
