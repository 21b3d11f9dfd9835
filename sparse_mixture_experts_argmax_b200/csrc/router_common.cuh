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
    if (bidx >= N) {          // no finite maximum (non-finite logits): flag, keep in range
      bidx = 0;
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

// Routing of R <= 128 token rows (R a multiple of 32, NT = 256 threads) from fp32
// logits Z[R][zs] (bias added; columns N .. NP-1 hold -inf), with TPT = 256 / R
// threads per token, each holding NP / TPT logits: max/argmax (lowest index on
// ties), exp-sum and gate reduced over the token's thread group with shuffles;
// p overwrites Z in place.  In-block ranks: match_any over each warp's 32
// tokens, plus the counts of the earlier warps.  Per-expert counts and sums of
// p (rows in token order: deterministic).  Rows at or beyond ntok are skipped;
// a block that starts beyond the batch writes nothing.  Shared scratch: eid[R],
// wcnt[R/32][NP].  Every thread of the CTA (256) calls this.
template <int NP>
__device__ __forceinline__ void route_rows_grouped(float* Z, int zs, int R, int ntok, int t0,
                                                   int N, int b, int* __restrict__ expert_idx,
                                                   float* __restrict__ gate,
                                                   int* __restrict__ local_rank,
                                                   int* __restrict__ blk_count,
                                                   float* __restrict__ blk_psum, WsHeader* hdr,
                                                   int* eid, int* wcnt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tpt = 256 / R;                 // threads per token: 8, 4 or 2
  const int ept = NP / tpt;                // logits per thread
  const int i = tid / tpt, sub = tid % tpt;
  const bool valid = i < ntok;
  for (int k = tid; k < (R / 32) * NP; k += 256) wcnt[k] = 0;
  float* zr = Z + i * zs + sub * ept;
  float best = -INFINITY;
  int bidx = 0x7fffffff;
  if (valid) {
    for (int j = 0; j < ept; ++j) {
      const float v = zr[j];
      if (v > best) { best = v; bidx = sub * ept + j; }
    }
  }
  for (int off = 1; off < tpt; off <<= 1) {   // the group's lanes are consecutive
    const float ov = __shfl_xor_sync(0xffffffffu, best, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
    if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
  }
  float ssum = 0.f;
  if (valid) {
    for (int j = 0; j < ept; ++j) {
      const float e = (sub * ept + j < N) ? expf(zr[j] - best) : 0.f;
      zr[j] = e;
      ssum += e;
    }
  }
  for (int off = 1; off < tpt; off <<= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, off);
  const float inv = 1.0f / ssum;
  if (valid) {
    for (int j = 0; j < ept; ++j) zr[j] *= inv;
    if (bidx >= N) {          // no finite maximum (non-finite logits): flag, keep in range
      bidx = 0;
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
    for (int w = 0; w < R / 32; ++w) c += wcnt[w * NP + n];
    cnt_row[n] = c;
    float a = 0.f;
    for (int r = 0; r < ntok; ++r) a += Z[r * zs + n];
    ps_row[n] = a;
  }
}

}  // namespace swl
