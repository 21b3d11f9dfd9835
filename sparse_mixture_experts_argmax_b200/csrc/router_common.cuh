// Device code shared by the router kernels: the per-token softmax / argmax on a
// block of logit rows held in shared memory, and the block bookkeeping the
// dispatch scan consumes (Switch Transformer, explained, "Router" and recipe
// step 3: top-1 routing with slots claimed in token order).
#pragma once

#include <cuda_runtime.h>

#include "kernels.h"

namespace swl {

// Block-level bookkeeping: in-block stable rank of each token among the block's
// earlier tokens with the same expert, and the block's per-expert token counts
// (written by the first token of each expert).  eid[i] < 0 marks an absent
// token.  The caller zeroes the block's count row before and synchronises the
// block after.
__device__ __forceinline__ void block_ranks(const int* eid, int* lead_count, int ntok, int tpb,
                                            int t0, int* __restrict__ local_rank) {
  for (int i = threadIdx.x; i < tpb; i += blockDim.x) {
    const int e = eid[i];
    lead_count[i] = 0;
    if (e < 0) continue;
    int rank = 0;
    for (int j = 0; j < i; ++j) rank += (eid[j] == e);
    local_rank[t0 + i] = rank;
    if (rank == 0) {
      int c = 1;
      for (int j = i + 1; j < ntok; ++j) c += (eid[j] == e);
      lead_count[i] = c;
    }
  }
}

// Top-2 form of block_ranks: token i of the block holds assignments to experts
// eid1[i] (first choice) and eid2[i] (second; always a different expert).  The
// rank of assignment (i, k) is the number of earlier tokens of the block with
// an assignment to the same expert (token order, the dispatch mask's column
// cumsum), written to local_rank[2 (t0 + i) + k].  lead_count[i] (k = 0) /
// lead_count[tpb + i] (k = 1) is set on the block's first assignment to an
// expert to that expert's number of assignments in the block, and lead_first[i]
// on a token that is the first with that expert as FIRST choice to the number
// of first choices of it.  eid1[i] < 0 marks an absent token.
__device__ __forceinline__ void block_ranks_top2(const int* eid1, const int* eid2,
                                                 int* lead_count, int* lead_first, int ntok,
                                                 int tpb, int t0, int* __restrict__ local_rank) {
  for (int i = threadIdx.x; i < tpb; i += blockDim.x) {
    lead_count[i] = 0;
    lead_count[tpb + i] = 0;
    lead_first[i] = 0;
    if (i >= ntok || eid1[i] < 0) continue;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int e = k == 0 ? eid1[i] : eid2[i];
      int rank = 0, first = 0;
      for (int j = 0; j < i; ++j) {
        rank += (eid1[j] == e) | (eid2[j] == e);
        first += (eid1[j] == e);
      }
      local_rank[2 * (t0 + i) + k] = rank;
      if (rank == 0) {
        int c = 1;
        for (int j = i + 1; j < ntok; ++j) c += (eid1[j] == e) | (eid2[j] == e);
        lead_count[k * tpb + i] = c;
      }
      if (k == 0 && first == 0) {
        int c = 1;
        for (int j = i + 1; j < ntok; ++j) c += (eid1[j] == e);
        lead_first[i] = c;
      }
    }
  }
}

// Routing of R token rows t0 .. t0+R-1 (dispatch block b) from fp32 logits Z
// (row stride zs; bias already added; columns N .. 32*NPL-1 hold -inf):
//   m = max_i z_i with the lowest index on ties; s = sum_i exp(z_i - m);
//   expert = argmax, gate = p at the argmax = 1/s; p_i = exp(z_i - m)/s.
// One warp per token (each lane holds NPL logits), warps take rows
// round-robin.  Then the block's ranks, per-expert counts and per-expert sums of
// p (each warp's rows in order, then warps in order: deterministic).  Rows at or
// beyond T (ntok = valid rows) are skipped; a block that starts at or beyond T
// writes nothing.  s_psum holds kWarps x 32*NPL floats; eid / lead_count R ints.
// Every thread of the CTA calls this.
template <int NPL, int kWarps>
__device__ __forceinline__ void route_rows(const float* Z, int zs, int R, int ntok, int t0, int N,
                                           int b, int* __restrict__ expert_idx,
                                           float* __restrict__ gate, int* __restrict__ local_rank,
                                           int* __restrict__ blk_count,
                                           float* __restrict__ blk_psum, WsHeader* hdr, int* eid,
                                           int* lead_count, float* s_psum) {
  constexpr int BN = 32 * NPL;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float pacc[NPL];
#pragma unroll
  for (int j = 0; j < NPL; ++j) pacc[j] = 0.f;
  for (int i = warp; i < R; i += kWarps) {
    if (i >= ntok) {
      if (lane == 0) eid[i] = -1;
      continue;
    }
    float v[NPL];
#pragma unroll
    for (int j = 0; j < NPL; ++j) v[j] = Z[i * zs + lane + 32 * j];
    float best = -INFINITY;
    int bidx = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NPL; ++j)
      if (v[j] > best) { best = v[j]; bidx = lane + 32 * j; }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
      if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
    }
    float ssum = 0.f;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      v[j] = (lane + 32 * j < N) ? expf(v[j] - best) : 0.f;
      ssum += v[j];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, off);
    const float inv = 1.0f / ssum;
#pragma unroll
    for (int j = 0; j < NPL; ++j) pacc[j] += v[j] * inv;
    // a non-finite logit (NaN, or an infinite maximum that makes the exp sum
    // NaN) is flagged; an index with no finite maximum is kept in range
    if (bidx >= N || !isfinite(best) || !isfinite(ssum)) {
      if (bidx >= N) bidx = 0;
      if (lane == 0) atomicExch(&hdr->err, kDevNonFiniteLogits);
    }
    if (lane == 0) {
      expert_idx[t0 + i] = bidx;
      gate[t0 + i] = inv;       // p at the argmax: exp(0) / s
      eid[i] = bidx;
    }
  }
#pragma unroll
  for (int j = 0; j < NPL; ++j) s_psum[warp * BN + lane + 32 * j] = pacc[j];
  __syncthreads();
  if (ntok <= 0) return;      // block b lies beyond the batch: no row of its own
  block_ranks(eid, lead_count, ntok, R, t0, local_rank);
  int* cnt_row = blk_count + (size_t)b * N;
  float* ps_row = blk_psum + (size_t)b * N;
  for (int n = tid; n < N; n += kWarps * 32) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) a += s_psum[w * BN + n];
    ps_row[n] = a;
    cnt_row[n] = 0;
  }
  __syncthreads();
  for (int i = tid; i < ntok; i += kWarps * 32) {
    if (lead_count[i] > 0) cnt_row[eid[i]] = lead_count[i];
  }
}

// Routing of R token rows (R = 128, 64 or 32; 256 threads) from fp32 logits
// Z[R][zs] (bias added; columns N .. NP-1 hold -inf), TPT = 256 / R threads per
// token.  Thread `sub` of a token's group holds the columns sub, sub + TPT, ...
// in registers: max/argmax (lowest index on ties) and exp-sum in four
// interleaved partial chains, then reduced over the group with shuffles; gate =
// 1 / sum; p overwrites Z in place.  With zs = NP + TPT (mod 32)
// the group's lanes read 32 distinct banks.  In-block ranks: match_any over
// each warp's 32 tokens, plus the counts of the earlier warps.  Per-expert
// counts, and per-expert sums of p over the rows in a fixed order (contiguous
// row ranges summed in parallel, then the ranges in order: deterministic).
// Rows at or beyond ntok are skipped; a block that starts beyond the batch
// writes nothing.  Shared scratch: eid[R], wcnt[R/32][NP], red[256].  Every
// thread of the CTA (256) calls this.
template <int NP, int R>
__device__ __forceinline__ void route_rows_grouped(float* Z, int zs, int ntok, int t0, int N,
                                                   int b, int* __restrict__ expert_idx,
                                                   float* __restrict__ gate,
                                                   int* __restrict__ local_rank,
                                                   int* __restrict__ blk_count,
                                                   float* __restrict__ blk_psum, WsHeader* hdr,
                                                   int* eid, int* wcnt, float* red) {
  static_assert(R == 128 || R == 64 || R == 32, "tile rows");
  constexpr int TPT = 256 / R;             // threads per token: 2, 4 or 8
  constexpr int EPT = NP / TPT;            // logits per thread
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i = tid / TPT, sub = tid % TPT;
  const bool valid = i < ntok;
  for (int k = tid; k < (R / 32) * NP; k += 256) wcnt[k] = 0;
  float* zr = Z + i * zs + sub;
  static_assert(EPT % 4 == 0, "four interleaved partial maxima and sums");
  float v[EPT];
  // four independent max/argmax chains (column j goes to chain j % 4; each
  // keeps its lowest index among equal maxima), then merged the same way
  float bq[4];
  int iq[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) { bq[q] = -INFINITY; iq[q] = 0x7fffffff; }
  if (valid) {
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      v[j] = zr[j * TPT];
      if (v[j] > bq[j & 3]) { bq[j & 3] = v[j]; iq[j & 3] = sub + j * TPT; }
    }
  }
  float best = bq[0];
  int bidx = iq[0];
#pragma unroll
  for (int q = 1; q < 4; ++q)
    if (bq[q] > best || (bq[q] == best && iq[q] < bidx)) { best = bq[q]; bidx = iq[q]; }
#pragma unroll
  for (int off = 1; off < TPT; off <<= 1) {   // the group's lanes are consecutive
    const float ov = __shfl_xor_sync(0xffffffffu, best, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
    if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
  }
  // the padded columns hold -inf: exp gives exactly 0 there, with no branch
  // per column (a finite maximum exists unless the row is flagged below)
  float sq[4] = {0.f, 0.f, 0.f, 0.f};
  if (valid) {
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      v[j] = expf(v[j] - best);
      sq[j & 3] += v[j];
    }
  }
  float ssum = (sq[0] + sq[1]) + (sq[2] + sq[3]);
#pragma unroll
  for (int off = 1; off < TPT; off <<= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, off);
  const float inv = 1.0f / ssum;
  if (valid) {
#pragma unroll
    for (int j = 0; j < EPT; ++j) zr[j * TPT] = v[j] * inv;
    // a non-finite logit (NaN, or an infinite maximum that makes the exp sum
    // NaN) is flagged; an index with no finite maximum is kept in range
    if (bidx >= N || !isfinite(best) || !isfinite(ssum)) {
      if (bidx >= N) bidx = 0;
      if (sub == 0) atomicExch(&hdr->err, kDevNonFiniteLogits);
    }
    if (sub == 0) {
      expert_idx[t0 + i] = bidx;
      gate[t0 + i] = inv;     // p at the argmax: exp(0) / s
    }
  }
  if (sub == 0) eid[i] = valid ? bidx : -1;
  __syncthreads();
  if (ntok <= 0) return;      // block b lies beyond the batch: no row of its own
  // in-block ranks: warp w takes tokens [32w, 32w + 32)
  int e = -1;
  unsigned int mask = 0u;
  const unsigned int lanes_below = (1u << lane) - 1u;
  if (warp < R / 32) {
    e = eid[warp * 32 + lane];
    mask = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (mask & lanes_below) == 0u) wcnt[warp * NP + e] = __popc(mask);
  }
  // partial sums of p: thread (g, n) adds rows [g*RPG, g*RPG + RPG) of column n
  constexpr int G = 256 / NP;
  constexpr int RPG = (R + G - 1) / G;
  {
    const int g = tid / NP, n = tid % NP;
    if (g < G) {
      float acc = 0.f;
      const int r0 = g * RPG, r1 = min(ntok, r0 + RPG);
      if (r1 - r0 == RPG) {     // full range: loads issued ahead of the adds
#pragma unroll
        for (int rr = 0; rr < RPG; ++rr) acc += Z[(r0 + rr) * zs + n];
      } else {
        for (int rr = r0; rr < r1; ++rr) acc += Z[rr * zs + n];
      }
      red[g * NP + n] = acc;
    }
  }
  __syncthreads();
  if (warp < R / 32 && e >= 0) {
    int rank = __popc(mask & lanes_below);
    for (int w = 0; w < warp; ++w) rank += wcnt[w * NP + e];
    local_rank[t0 + warp * 32 + lane] = rank;
  }
  int* cnt_row = blk_count + (size_t)b * N;
  float* ps_row = blk_psum + (size_t)b * N;
  for (int n = tid; n < N; n += 256) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < R / 32; ++w) c += wcnt[w * NP + n];
    cnt_row[n] = c;
    float a = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) a += red[g * NP + n];
    ps_row[n] = a;
  }
}

}  // namespace swl
