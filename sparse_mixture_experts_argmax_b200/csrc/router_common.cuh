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

}  // namespace swl
