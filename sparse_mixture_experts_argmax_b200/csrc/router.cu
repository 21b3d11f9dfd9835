// Router of the Switch layer, in fp32 ("selective precision": the router input
// is cast to float32 and logits, softmax and the argmax are computed in fp32;
// paper-graph summary of arXiv 2101.03961, section 3.4 "The selective precision
// solution"; Switch Transformer, explained, recipe step 2).
//
//   logits  z_t = W_r x_t (+ b_r)            "The mathematics of routing": h(x) = W_r x
//   probs   p_t = softmax(z_t)                p_i = exp(h_i) / sum_j exp(h_j)
//   choice  e_t = argmax_i p_t,i (lowest index on ties), gate g_t = p_t,e_t
//
// Stage 1 (router_logits_kernel): register-tiled fp32 FFMA GEMM [T,d] x [N,d]^T,
//   K split into slices when T*N alone would not fill the GPU.
// Stage 2 (router_softmax_kernel): one CTA per block of tokens; one warp per
//   token row (held in registers) for max/argmax/sum via warp shuffles; then, per
//   block, the in-block rank of every token among the block's tokens with the
//   same expert, the block's per-expert token counts, and per-expert sums of p.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "router_common.cuh"
#include "sm100_ptx.cuh"

namespace cg = cooperative_groups;



namespace swl {
namespace {

constexpr int kBK = 16;

__device__ __forceinline__ void load8(const float* row, int k, int d, bool vec_ok, float (&v)[8]) {
  if (vec_ok && k + 8 <= d) {
    const float4 a = *reinterpret_cast<const float4*>(row + k);
    const float4 b = *reinterpret_cast<const float4*>(row + k + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = (k + j < d) ? row[k + j] : 0.f;
  }
}

__device__ __forceinline__ void load8(const __nv_bfloat16* row, int k, int d, bool vec_ok,
                                      float (&v)[8]) {
  if (vec_ok && k + 8 <= d) {
    const uint4 u = *reinterpret_cast<const uint4*>(row + k);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h[j]);
      v[2 * j] = f.x;
      v[2 * j + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = (k + j < d) ? __bfloat162float(row[k + j]) : 0.f;
  }
}

// Main loop of one logits tile: acc[i][j] = sum_{k in [k_lo, k_hi)} x[m0 + ty*8 + i, k] *
// W_r[n(j), k] with n(j) = n0 + tx*4 + j for j < 4 and n0 + BN/2 + tx*4 + (j-4) for
// j >= 4 (the two halves keep the float4 reads of a quarter-warp on distinct banks).  THREADS = (BM/8)*(BN/8) threads with 8 x 8 outputs each; K
// staged through shared memory (As[2][kBK][BM], Bs[2][kBK][BN], transposed so the
// inner loop reads float4 vectors) in chunks of 16 with register prefetch of the
// next chunk.  Rows >= T, experts >= N and k >= k_hi read as zero.
template <typename TX, int BM, int BN>
__device__ __forceinline__ void logits_mainloop(const TX* __restrict__ x,
                                                const float* __restrict__ W_r, int T, int d, int N,
                                                int m0, int n0, int k_lo, int k_hi,
                                                float (*As)[kBK][BM], float (*Bs)[kBK][BN],
                                                float (&acc)[8][8]) {
  constexpr int kThreads = (BM / 8) * (BN / 8);
  const int tid = threadIdx.x;
  const int tx = tid % (BN / 8);
  const int ty = tid / (BN / 8);
  const bool xvec = ((d * (int)sizeof(TX)) % 16 == 0) &&
                    ((reinterpret_cast<uintptr_t>(x) & 15) == 0);
  const bool wvec = ((d % 4) == 0) && ((reinterpret_cast<uintptr_t>(W_r) & 15) == 0);

  constexpr int A_SLOTS = BM * 2;   // (token, k-half) pairs per chunk
  constexpr int B_SLOTS = BN * 2;
  constexpr int A_PER = (A_SLOTS + kThreads - 1) / kThreads;
  constexpr int B_PER = (B_SLOTS + kThreads - 1) / kThreads;
  float ra[A_PER][8];
  float rb[B_PER][8];

  auto gload = [&](int k0) {
#pragma unroll
    for (int i = 0; i < A_PER; ++i) {
      const int s = tid + i * kThreads;
      if (s < A_SLOTS) {
        const int m = s % BM, kh = s / BM;
        const int t = m0 + m;
        if (t < T) {
          load8(x + (size_t)t * d, k0 + kh * 8, k_hi, xvec, ra[i]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) ra[i][j] = 0.f;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < B_PER; ++i) {
      const int s = tid + i * kThreads;
      if (s < B_SLOTS) {
        const int n = s % BN, kh = s / BN;
        if (n0 + n < N) {
          load8(W_r + (size_t)(n0 + n) * d, k0 + kh * 8, k_hi, wvec, rb[i]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) rb[i][j] = 0.f;
        }
      }
    }
  };
  auto sstore = [&](int buf) {
#pragma unroll
    for (int i = 0; i < A_PER; ++i) {
      const int s = tid + i * kThreads;
      if (s < A_SLOTS) {
        const int m = s % BM, kh = s / BM;
#pragma unroll
        for (int j = 0; j < 8; ++j) As[buf][kh * 8 + j][m] = ra[i][j];
      }
    }
#pragma unroll
    for (int i = 0; i < B_PER; ++i) {
      const int s = tid + i * kThreads;
      if (s < B_SLOTS) {
        const int n = s % BN, kh = s / BN;
#pragma unroll
        for (int j = 0; j < 8; ++j) Bs[buf][kh * 8 + j][n] = rb[i][j];
      }
    }
  };

#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int nk = (k_hi - k_lo + kBK - 1) / kBK;
  if (nk <= 0) return;
  gload(k_lo);
  sstore(0);
  __syncthreads();
  for (int kc = 0; kc < nk; ++kc) {
    const int buf = kc & 1;
    if (kc + 1 < nk) gload(k_lo + (kc + 1) * kBK);
#pragma unroll
    for (int k = 0; k < kBK; ++k) {
      float a[8], b[8];
      *reinterpret_cast<float4*>(&a[0]) = *reinterpret_cast<const float4*>(&As[buf][k][ty * 8]);
      *reinterpret_cast<float4*>(&a[4]) =
          *reinterpret_cast<const float4*>(&As[buf][k][ty * 8 + 4]);
      *reinterpret_cast<float4*>(&b[0]) = *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 4]);
      *reinterpret_cast<float4*>(&b[4]) =
          *reinterpret_cast<const float4*>(&Bs[buf][k][BN / 2 + tx * 4]);
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (kc + 1 < nk) sstore(buf ^ 1);
    __syncthreads();
  }
}

// Partial logits over one K slice: zpart[ks][t][n] = sum_{k in slice ks} x[t,k] W_r[n,k]
// (used when N is too wide for one CTA to hold a token's whole row; the softmax
// kernel adds the slices in order, then the bias).
template <typename TX, int BM, int BN>
__global__ void __launch_bounds__((BM / 8) * (BN / 8))
router_logits_kernel(const TX* __restrict__ x, const float* __restrict__ W_r,
                     float* __restrict__ zpart, int T, int d, int N, int kslice,
                     WsHeader* hdr) {
  __shared__ __align__(16) float As[2][kBK][BM];
  __shared__ __align__(16) float Bs[2][kBK][BN];
  pdl_trigger();
  pdl_wait();
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) {
    hdr->err = kDevOk;   // per-call device status
    hdr->done = 0u;      // arrival counter of the dispatch scan
  }
  const int tx = threadIdx.x % (BN / 8);
  const int ty = threadIdx.x / (BN / 8);
  const int m0 = blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  const int k_lo = blockIdx.z * kslice;
  const int k_hi = min(d, k_lo + kslice);
  float acc[8][8];
  logits_mainloop<TX, BM, BN>(x, W_r, T, d, N, m0, n0, k_lo, k_hi, As, Bs, acc);

  // lane tx holds experts n0 + tx*4 + {0..3} and n0 + BN/2 + tx*4 + {0..3}
  float* zs = zpart + (size_t)blockIdx.z * T * N;
  const bool vec_out = (N % 4) == 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = m0 + ty * 8 + i;
    if (t >= T) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int nb = n0 + h * (BN / 2) + tx * 4;
      float* zr = zs + (size_t)t * N + nb;
      if (vec_out && nb + 4 <= N) {
        *reinterpret_cast<float4*>(zr) =
            make_float4(acc[i][4 * h], acc[i][4 * h + 1], acc[i][4 * h + 2], acc[i][4 * h + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (nb + j < N) zr[j] = acc[i][4 * h + j];
      }
    }
  }
}

constexpr int kSoftmaxThreads = 256;
constexpr int kSoftmaxWarps = kSoftmaxThreads / 32;

// Order of (value, expert) pairs for the top-2 choice: larger value first,
// lower expert index first among equal values.
__device__ __forceinline__ bool rank_before(float v, int i, float w, int j) {
  return v > w || (v == w && i < j);
}

// (b1, i1) >= (b2, i2) and (c1, j1) >= (c2, j2) in the (value desc, index asc)
// order: the two largest of the four, in order, into (b1, i1), (b2, i2).
__device__ __forceinline__ void top2_merge(float& b1, int& i1, float& b2, int& i2, float c1,
                                           int j1, float c2, int j2) {
  if (rank_before(c1, j1, b1, i1)) {
    if (rank_before(b1, i1, c2, j2)) { b2 = b1; i2 = i1; } else { b2 = c2; i2 = j2; }
    b1 = c1;
    i1 = j1;
  } else if (rank_before(c1, j1, b2, i2)) {
    b2 = c1;
    i2 = j1;
  }
}


// One CTA per block of tpb tokens; one warp per token with the row of logits
// held in registers (NPL = logits per lane, N <= 32*NPL):
//   z = sum of the K-slice partials + b_r; m = max with the lowest index;
//   s = sum exp(z - m); gate = p at the argmax = 1/s; p_i = exp(z_i - m)/s is
//   accumulated per lane into per-expert sums.
// Then per block: ranks, counts blk_count[b][e], probability sums blk_psum[b][e]
// (each warp's tokens in order, warps in order).  TOP2: as the streaming
// kernel's top-2 form (below), with [T, 2] outputs.
template <int NPL, bool TOP2>
__global__ void __launch_bounds__(kSoftmaxThreads)
router_softmax_kernel(const float* __restrict__ zpart, int nsplit, const float* __restrict__ b_r,
                      int T, int N, int tpb, int* __restrict__ expert_idx,
                      float* __restrict__ gate, int* __restrict__ local_rank,
                      int* __restrict__ blk_count, float* __restrict__ blk_psum,
                      int* __restrict__ blk_count1, int normalize, WsHeader* hdr) {
  constexpr int K = TOP2 ? 2 : 1;
  extern __shared__ float smem_f[];
  float* s_bias = smem_f;                 // [N]
  float* s_psum = smem_f + N;             // [kSoftmaxWarps][N]
  __shared__ int eid[K][kTokensPerBlock];
  __shared__ int lead_count[K * kTokensPerBlock];
  __shared__ int lead_first[TOP2 ? kTokensPerBlock : 1];
  pdl_trigger();
  pdl_wait();   // partial logits come from the logits kernel
  const int b = blockIdx.x;
  const int t0 = b * tpb;
  const int ntok = min(tpb, T - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int n = threadIdx.x; n < N; n += kSoftmaxThreads) s_bias[n] = b_r ? b_r[n] : 0.f;
  __syncthreads();

  float acc[NPL];
#pragma unroll
  for (int j = 0; j < NPL; ++j) acc[j] = 0.f;
  const size_t slice = (size_t)T * N;
  for (int i = warp; i < tpb; i += kSoftmaxWarps) {
    if (i >= ntok) {
      if (lane == 0) {
        eid[0][i] = -1;
        eid[K - 1][i] = -1;
      }
      continue;
    }
    const int t = t0 + i;
    const float* row = zpart + (size_t)t * N;
    // all loads of a slice are issued before any is used (one round trip per slice)
    float v[NPL];
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const int n = lane + 32 * j;
      v[j] = (n < N) ? row[n] : 0.f;
    }
    for (int s = 1; s < nsplit; ++s) {
      float u[NPL];
#pragma unroll
      for (int j = 0; j < NPL; ++j) {
        const int n = lane + 32 * j;
        u[j] = (n < N) ? row[s * slice + n] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < NPL; ++j) v[j] += u[j];
    }
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const int n = lane + 32 * j;
      v[j] = (n < N) ? v[j] + s_bias[n] : -INFINITY;
    }
    float best = -INFINITY, second = -INFINITY;
    int bidx = 0x7fffffff, sidx = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {     // ascending columns: strict compares keep the lowest index
      if (v[j] > best) {
        if (TOP2) { second = best; sidx = bidx; }
        best = v[j];
        bidx = lane + 32 * j;
      } else if (TOP2 && v[j] > second) {
        second = v[j];
        sidx = lane + 32 * j;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
      if (TOP2) {
        const float os = __shfl_xor_sync(0xffffffffu, second, off);
        const int oj = __shfl_xor_sync(0xffffffffu, sidx, off);
        top2_merge(best, bidx, second, sidx, ov, oi, os, oj);
      } else if (ov > best || (ov == best && oi < bidx)) {
        best = ov;
        bidx = oi;
      }
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
    for (int j = 0; j < NPL; ++j) acc[j] += v[j] * inv;
    // a non-finite logit (NaN, or an infinite maximum that makes the exp sum
    // NaN) is flagged; an index with no finite maximum is kept in range
    bool bad = bidx >= N || !isfinite(best) || !isfinite(ssum);
    if (bidx >= N) bidx = 0;
    if (TOP2) {
      bad = bad || sidx >= N || sidx == bidx;
      if (sidx >= N || sidx == bidx) sidx = bidx == 0 ? 1 : 0;
    }
    if (bad && lane == 0) atomicExch(&hdr->err, kDevNonFiniteLogits);
    if (lane == 0) {
      if (TOP2) {
        const float e2 = expf(second - best);      // p_e2 / p_e1
        expert_idx[2 * t] = bidx;
        expert_idx[2 * t + 1] = sidx;
        gate[2 * t] = normalize ? 1.0f / (1.0f + e2) : inv;
        gate[2 * t + 1] = normalize ? e2 / (1.0f + e2) : e2 * inv;
        eid[0][i] = bidx;
        eid[K - 1][i] = sidx;
      } else {
        expert_idx[t] = bidx;
        gate[t] = inv;            // p at the argmax: exp(0) / s
        eid[0][i] = bidx;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < NPL; ++j) {
    const int n = lane + 32 * j;
    if (n < N) s_psum[warp * N + n] = acc[j];
  }
  __syncthreads();
  if (TOP2) {
    block_ranks_top2(eid[0], eid[K - 1], lead_count, lead_first, ntok, tpb, t0, local_rank);
  } else {
    block_ranks(eid[0], lead_count, ntok, tpb, t0, local_rank);
  }
  int* cnt_row = blk_count + (size_t)b * N;
  int* cnt1_row = TOP2 ? blk_count1 + (size_t)b * N : nullptr;
  float* ps_row = blk_psum + (size_t)b * N;
  for (int n = threadIdx.x; n < N; n += kSoftmaxThreads) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kSoftmaxWarps; ++w) a += s_psum[w * N + n];
    ps_row[n] = a;
    cnt_row[n] = 0;
    if (TOP2) cnt1_row[n] = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ntok; i += kSoftmaxThreads) {
    if (lead_count[i] > 0) cnt_row[eid[0][i]] = lead_count[i];
    if (TOP2) {
      if (lead_count[tpb + i] > 0) cnt_row[eid[K - 1][i]] = lead_count[tpb + i];
      if (lead_first[i] > 0) cnt1_row[eid[0][i]] = lead_first[i];
    }
  }
}

// Same contract for any N (rows streamed from memory, three passes): the
// combined logits are written back into slice 0, which then holds p.
__global__ void __launch_bounds__(kSoftmaxThreads)
router_softmax_wide_kernel(float* __restrict__ zpart, int nsplit, const float* __restrict__ b_r,
                           int T, int N, int tpb, int* __restrict__ expert_idx,
                           float* __restrict__ gate, int* __restrict__ local_rank,
                           int* __restrict__ blk_count, float* __restrict__ blk_psum,
                           WsHeader* hdr) {
  __shared__ int eid[kTokensPerBlock];
  __shared__ int lead_count[kTokensPerBlock];
  pdl_trigger();
  pdl_wait();   // partial logits come from the logits kernel
  const int b = blockIdx.x;
  const int t0 = b * tpb;
  const int ntok = min(tpb, T - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t slice = (size_t)T * N;

  for (int i = warp; i < tpb; i += kSoftmaxWarps) {
    if (i >= ntok) {
      if (lane == 0) eid[i] = -1;
      continue;
    }
    const int t = t0 + i;
    float* row = zpart + (size_t)t * N;
    float best = -INFINITY;
    int bidx = 0x7fffffff;
    for (int j = lane; j < N; j += 32) {
      float v = row[j];
      for (int s = 1; s < nsplit; ++s) v += row[s * slice + j];
      v += b_r ? b_r[j] : 0.f;
      row[j] = v;
      if (v > best) { best = v; bidx = j; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
      if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
    }
    float ssum = 0.f;
    for (int j = lane; j < N; j += 32) {
      const float e = expf(row[j] - best);
      row[j] = e;
      ssum += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, off);
    const float inv = 1.0f / ssum;
    for (int j = lane; j < N; j += 32) row[j] *= inv;
    // a non-finite logit (NaN, or an infinite maximum that makes the exp sum
    // NaN) is flagged; an index with no finite maximum is kept in range
    if (bidx >= N || !isfinite(best) || !isfinite(ssum)) {
      if (bidx >= N) bidx = 0;
      if (lane == 0) atomicExch(&hdr->err, kDevNonFiniteLogits);
    }
    if (lane == 0) {
      expert_idx[t] = bidx;
      gate[t] = inv;
      eid[i] = bidx;
    }
  }
  __syncthreads();
  block_ranks(eid, lead_count, ntok, tpb, t0, local_rank);
  int* cnt_row = blk_count + (size_t)b * N;
  float* ps_row = blk_psum + (size_t)b * N;
  for (int e = threadIdx.x; e < N; e += kSoftmaxThreads) {
    float a = 0.f;
    const float* col = zpart + (size_t)t0 * N + e;
    for (int i = 0; i < ntok; ++i) a += col[(size_t)i * N];
    ps_row[e] = a;
    cnt_row[e] = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ntok; i += kSoftmaxThreads) {
    if (lead_count[i] > 0) cnt_row[eid[i]] = lead_count[i];
  }
}

// Streaming softmax for N > 128 whose logits come in one slice (ksplit = 1)
// with N % 4 == 0: a persistent CTA per SM takes dispatch blocks b =
// blockIdx.x, blockIdx.x + gridDim.x, ...  Its 16 warps form row groups of WPR
// warps (one warp per token row up to N = 1024, two up to 2048); group g takes
// rows g, g + G, ... of each block (G = 16 / WPR groups) and runs on its own:
// its leader streams each of its rows into a private ring of kStreamStages
// row buffers with one bulk copy (cp.async.bulk) per row, so the next rows are
// in flight while one is processed, and the only waits between warps are the
// group's own (a named barrier when WPR = 2) and one block-wide barrier per
// block.  Per row, each warp holds its part of the float4 columns in registers
// (+ b_r when there is one):
//   the maximum m (fmax in four chains, warp shuffles, the group's parts);
//   the expert: the lowest column holding m (equal values keep the lowest
//     index), found by comparing against m and a warp minimum;
//   e = 2^(z log2 e - m log2 e) and its sum s; gate = 1/s (p at the expert);
//   p = e/s added to the warp's per-column sums for the block (registers:
//     a warp sees the same columns on every row).
// At the end of a block the groups' column sums are added in group order
// (deterministic), then the in-block ranks and per-expert counts are written.
constexpr int kStreamThreads = 512;
constexpr int kStreamWarps = kStreamThreads / 32;
constexpr int kStreamStages = 3;                       // row buffers per row group
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ constexpr int stream_wpr(int N) { return N <= 1024 ? 1 : 2; }

__host__ __device__ constexpr size_t stream_softmax_smem(int N) {
  // every group's ring, then b_r and the block's column sums
  return 128 + (static_cast<size_t>(kStreamStages) * (kStreamWarps / stream_wpr(N)) + 2) * N *
                   sizeof(float);
}

// 2^x on the special-function unit (PTX ex2.approx.ftz: relative error near
// 2^-22; a result below the normal range is flushed to zero).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// TOP2: the first choice and the runner-up (lowest index on ties for both,
// two experts per token, see top2_merge), gates p_e1 and p_e2, divided by
// their sum when `normalize`; outputs are [T, 2] (first choice, then second),
// the block statistics count both choices (blk_count) and, for the aux loss,
// first choices alone (blk_count1).
// V4: float4 columns per lane, N <= 128 * WPR * V4; kFull: N == 128 * WPR * V4
// (every lane's columns exist: no range checks)
template <int V4, int WPR, bool TOP2, bool kFull>
__global__ void __launch_bounds__(kStreamThreads, 1)
router_softmax_stream_kernel(const float* __restrict__ z, const float* __restrict__ b_r, int T,
                             int N, int tpb, int nblk, int* __restrict__ expert_idx,
                             float* __restrict__ gate, int* __restrict__ local_rank,
                             int* __restrict__ blk_count, float* __restrict__ blk_psum,
                             int* __restrict__ blk_count1, int normalize, WsHeader* hdr,
                             unsigned long long wait_ns) {
  constexpr int G = kStreamWarps / WPR;   // row groups
  constexpr int S = kStreamStages;
  constexpr int K = TOP2 ? 2 : 1;
  extern __shared__ uint8_t smem_raw[];
  float* buf = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  float* s_bias = buf + static_cast<size_t>(G) * S * N;   // [N]
  float* s_psum = s_bias + N;                             // [N]
  __shared__ uint64_t full[G][S];
  __shared__ int eid[K][kTokensPerBlock];
  __shared__ int lead_count[K * kTokensPerBlock];
  __shared__ int lead_first[TOP2 ? kTokensPerBlock : 1];
  // per group and part: maximum (runner-up), their experts, the exp sum
  __shared__ float x_m[G][WPR], x_m2[G][WPR], x_s[G][WPR];
  __shared__ int x_h[G][WPR], x_h2[G][WPR];
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp / WPR, part = warp % WPR;
  const int NV = N >> 2;                       // float4 per row
  const int NVp = (NV + WPR - 1) / WPR;        // float4 per part
  const int q_lo = part * NVp, q_hi = min(NV, q_lo + NVp);
  const bool has_bias = b_r != nullptr;
  const bool leader = part == 0 && lane == 0;
  float* ring = buf + static_cast<size_t>(grp) * S * N;
  volatile int* ab = &s_abort;
  pdl_trigger();
  if (tid == 0) {
    for (int g = 0; g < G; ++g)
      for (int i = 0; i < S; ++i) ptx::mbar_init(&full[g][i], 1);
    s_abort = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
  }
  if (has_bias)
    for (int n = tid; n < N; n += kStreamThreads) s_bias[n] = b_r[n];
  __syncthreads();
  pdl_wait();   // the logits come from the logits kernel

  // the leader's cursor over its group's rows, in the consumers' order
  int pb = blockIdx.x, pr = grp, issued = 0;
  const uint32_t row_bytes = static_cast<uint32_t>(N) * 4u;
  auto issue_next = [&]() {
    while (pb < nblk && pr >= min(tpb, T - pb * tpb)) {
      pr = grp;
      pb += gridDim.x;
    }
    if (pb >= nblk) return;
    uint64_t* bar = &full[grp][issued % S];
    ptx::mbar_arrive_expect_tx(bar, row_bytes);
    ptx::bulk_load_g2s(ring + static_cast<size_t>(issued % S) * N,
                       z + (static_cast<size_t>(pb) * tpb + pr) * N, row_bytes, bar);
    ++issued;
    pr += G;
  };
  if (leader)
    for (int i = 0; i < S; ++i) issue_next();

  const float4* bias4 = reinterpret_cast<const float4*>(s_bias);
  int ci = 0;   // rows of this group consumed
  for (int b = blockIdx.x; b < nblk; b += gridDim.x) {
    const int t0b = b * tpb, ntb = min(tpb, T - t0b);
    float4 acc[V4];
#pragma unroll
    for (int k = 0; k < V4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = grp; r < ntb; r += G, ++ci) {
      const int slot = ci % S;
      // after a time-out every wait returns at once (the flag is shared), and
      // the loop still takes every barrier, so no warp is left waiting
      if (!ptx::mbar_wait(&full[grp][slot], static_cast<uint32_t>(ci / S) & 1u, ab, wait_ns))
        *ab = 1;
      const float4* row = reinterpret_cast<const float4*>(ring + static_cast<size_t>(slot) * N);
      float4 v[V4];
#pragma unroll
      for (int k = 0; k < V4; ++k) {
        const int q = q_lo + lane + 32 * k;
        if (kFull || q < q_hi) {
          float4 a = row[q];
          if (has_bias) {
            const float4 bb = bias4[q];
            a = make_float4(a.x + bb.x, a.y + bb.y, a.z + bb.z, a.w + bb.w);
          }
          v[k] = a;
        } else {
          v[k] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
      }
      float best, second = -INFINITY;
      int bidx = 0x7fffffff, sidx = 0x7fffffff;
      if constexpr (TOP2) {
        // chain c holds column 4q + c: ascending columns per chain, so a strict
        // compare keeps each chain's lowest index among equal values
        float bq[4], sq[4];
        int iq[4], jq[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          bq[c] = sq[c] = -INFINITY;
          iq[c] = jq[c] = 0x7fffffff;
        }
        auto insert = [&](int c, float val, int col) {
          if (val > bq[c]) {
            sq[c] = bq[c];
            jq[c] = iq[c];
            bq[c] = val;
            iq[c] = col;
          } else if (val > sq[c]) {
            sq[c] = val;
            jq[c] = col;
          }
        };
#pragma unroll
        for (int k = 0; k < V4; ++k) {
          const int q = q_lo + lane + 32 * k;
          insert(0, v[k].x, 4 * q);
          insert(1, v[k].y, 4 * q + 1);
          insert(2, v[k].z, 4 * q + 2);
          insert(3, v[k].w, 4 * q + 3);
        }
        best = bq[0];
        bidx = iq[0];
        second = sq[0];
        sidx = jq[0];
#pragma unroll
        for (int c = 1; c < 4; ++c) top2_merge(best, bidx, second, sidx, bq[c], iq[c], sq[c], jq[c]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, best, off);
          const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
          const float os = __shfl_xor_sync(0xffffffffu, second, off);
          const int oj = __shfl_xor_sync(0xffffffffu, sidx, off);
          top2_merge(best, bidx, second, sidx, ov, oi, os, oj);
        }
        if (WPR > 1) {
          if (lane == 0) {
            x_m[grp][part] = best;
            x_h[grp][part] = bidx;
            x_m2[grp][part] = second;
            x_h2[grp][part] = sidx;
          }
          ptx::named_bar_sync(1 + grp, 32 * WPR);
          best = x_m[grp][0];
          bidx = x_h[grp][0];
          second = x_m2[grp][0];
          sidx = x_h2[grp][0];
#pragma unroll
          for (int h = 1; h < WPR; ++h)
            top2_merge(best, bidx, second, sidx, x_m[grp][h], x_h[grp][h], x_m2[grp][h],
                       x_h2[grp][h]);
        }
      } else {
        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int k = 0; k < V4; ++k) {
          m0 = fmaxf(m0, v[k].x);
          m1 = fmaxf(m1, v[k].y);
          m2 = fmaxf(m2, v[k].z);
          m3 = fmaxf(m3, v[k].w);
        }
        const float lane_best = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
        best = lane_best;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, off));
        if (WPR > 1) {
          if (lane == 0) x_m[grp][part] = best;
          ptx::named_bar_sync(1 + grp, 32 * WPR);
          best = x_m[grp][0];
#pragma unroll
          for (int h = 1; h < WPR; ++h) best = fmaxf(best, x_m[grp][h]);
        }
        // the lowest column holding the maximum: searched only by the lanes
        // that hold it (columns in descending order, so the last match stands),
        // then the warp's minimum
        if (lane_best == best) {
#pragma unroll
          for (int k = V4 - 1; k >= 0; --k) {
            const int c4 = 4 * (q_lo + lane + 32 * k);
            if (v[k].w == best) bidx = c4 + 3;
            if (v[k].z == best) bidx = c4 + 2;
            if (v[k].y == best) bidx = c4 + 1;
            if (v[k].x == best) bidx = c4;
          }
        }
        bidx = static_cast<int>(__reduce_min_sync(0xffffffffu, static_cast<unsigned>(bidx)));
      }
      __syncwarp();
      // every warp of the group has its part in registers: the buffer is free
      if (leader && !*ab) {
        ptx::fence_proxy_async_smem();
        issue_next();
      }
      const float ml = best * kLog2e;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int k = 0; k < V4; ++k) {
        v[k].x = ex2_approx(fmaf(v[k].x, kLog2e, -ml));
        v[k].y = ex2_approx(fmaf(v[k].y, kLog2e, -ml));
        v[k].z = ex2_approx(fmaf(v[k].z, kLog2e, -ml));
        v[k].w = ex2_approx(fmaf(v[k].w, kLog2e, -ml));
        s0 += v[k].x;
        s1 += v[k].y;
        s2 += v[k].z;
        s3 += v[k].w;
      }
      float ssum = (s0 + s1) + (s2 + s3);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, off);
      if (WPR > 1) {
        if (lane == 0) {
          x_s[grp][part] = ssum;
          if (!TOP2) x_h[grp][part] = bidx;
        }
        ptx::named_bar_sync(1 + grp, 32 * WPR);
        ssum = x_s[grp][0];
        if (!TOP2) bidx = x_h[grp][0];
#pragma unroll
        for (int h = 1; h < WPR; ++h) {
          ssum += x_s[grp][h];
          if (!TOP2) bidx = min(bidx, x_h[grp][h]);
        }
      }
      const float inv = 1.0f / ssum;
#pragma unroll
      for (int k = 0; k < V4; ++k) {
        acc[k].x = fmaf(v[k].x, inv, acc[k].x);
        acc[k].y = fmaf(v[k].y, inv, acc[k].y);
        acc[k].z = fmaf(v[k].z, inv, acc[k].z);
        acc[k].w = fmaf(v[k].w, inv, acc[k].w);
      }
      if (leader) {
        // a non-finite logit (NaN, or an infinite maximum that makes the exp
        // sum NaN) is flagged; an index with no finite maximum is kept in range
        bool bad = bidx >= N || !isfinite(best) || !isfinite(ssum);
        if (bidx >= N) bidx = 0;
        if (TOP2) {
          bad = bad || sidx >= N || sidx == bidx;
          if (sidx >= N || sidx == bidx) sidx = bidx == 0 ? 1 : 0;
        }
        if (bad) atomicExch(&hdr->err, kDevNonFiniteLogits);
        const int t = t0b + r;
        if (TOP2) {
          const float e2 = exp2f((second - best) * kLog2e);   // p_e2 / p_e1
          expert_idx[2 * t] = bidx;
          expert_idx[2 * t + 1] = sidx;
          gate[2 * t] = normalize ? 1.0f / (1.0f + e2) : inv;
          gate[2 * t + 1] = normalize ? e2 / (1.0f + e2) : e2 * inv;
          eid[0][r] = bidx;
          eid[K - 1][r] = sidx;
        } else {
          expert_idx[t] = bidx;
          gate[t] = inv;          // p at the expert: 2^0 / s
          eid[0][r] = bidx;
        }
      }
    }
    // the block's sums of p: the groups' registers added in group order
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
      __syncthreads();
      if (grp == g) {
#pragma unroll
        for (int k = 0; k < V4; ++k) {
          const int q = q_lo + lane + 32 * k;
          if (kFull || q < q_hi) {
            float4* d = reinterpret_cast<float4*>(s_psum) + q;
            if (g == 0) {
              *d = acc[k];
            } else {
              const float4 o = *d;
              *d = make_float4(o.x + acc[k].x, o.y + acc[k].y, o.z + acc[k].z, o.w + acc[k].w);
            }
          }
        }
      }
    }
    __syncthreads();
    // block bookkeeping: ranks, the block's per-expert counts and sums of p
    if (TOP2) {
      block_ranks_top2(eid[0], eid[K - 1], lead_count, lead_first, ntb, ntb, t0b, local_rank);
    } else {
      block_ranks(eid[0], lead_count, ntb, ntb, t0b, local_rank);
    }
    int* cnt_row = blk_count + static_cast<size_t>(b) * N;
    int* cnt1_row = TOP2 ? blk_count1 + static_cast<size_t>(b) * N : nullptr;
    float4* ps_row = reinterpret_cast<float4*>(blk_psum + static_cast<size_t>(b) * N);
    for (int q = tid; q < NV; q += kStreamThreads) {
      ps_row[q] = reinterpret_cast<const float4*>(s_psum)[q];
      reinterpret_cast<int4*>(cnt_row)[q] = make_int4(0, 0, 0, 0);
      if (TOP2) reinterpret_cast<int4*>(cnt1_row)[q] = make_int4(0, 0, 0, 0);
    }
    __syncthreads();
    for (int i = tid; i < ntb; i += kStreamThreads) {
      if (lead_count[i] > 0) cnt_row[eid[0][i]] = lead_count[i];
      if (TOP2) {
        if (lead_count[ntb + i] > 0) cnt_row[eid[K - 1][i]] = lead_count[ntb + i];
        if (lead_first[i] > 0) cnt1_row[eid[0][i]] = lead_first[i];
      }
    }
    __syncthreads();   // eid / lead_count are reused by the next block
  }
  __syncthreads();
  if (*ab) {
    if (tid == 0) atomicExch(&hdr->err, kDevPipelineTimeout);
    // every issued copy must land before the CTA's shared memory goes away:
    // the last one issued into each buffer
    if (leader) {
      volatile int never = 0;
      for (int j = max(0, issued - S); j < issued; ++j)
        ptx::mbar_wait(&full[grp][j % S], static_cast<uint32_t>(j / S) & 1u, &never, wait_ns);
    }
    __syncthreads();
  }
}

// Warp-split router for small T and N <= BN (BN = 32, 64 or 128): logits,
// softmax, argmax and the block statistics in one kernel, one CTA per tile of
// TM = 2048/BN tokens.
// The 8 warps split K: warp w accumulates the whole TM x BN tile over the
// K chunks c = w, w+8, ... (8 x 8 register outer products per lane, staged
// through warp-private shared memory, so the main loop has no block barrier).
// The 8 partial tiles are then summed in warp order (deterministic), the bias
// added, and each token's softmax run by one warp.  The tile's TM tokens form
// one token block of the dispatch statistics.
template <typename TX, int BN>
__global__ void __launch_bounds__(256)
router_warpsplit_kernel(const TX* __restrict__ x, const float* __restrict__ W_r,
                    const float* __restrict__ b_r, int T, int d, int N,
                    int* __restrict__ expert_idx, float* __restrict__ gate,
                    int* __restrict__ local_rank, int* __restrict__ blk_count,
                    float* __restrict__ blk_psum, WsHeader* hdr) {
  constexpr int kWarps = 8;
  constexpr int TM = 2048 / BN;                 // tokens per tile
  constexpr int KC = BN <= 64 ? 16 : 8;         // K per chunk
  constexpr int TXN = BN / 8;                   // lanes along the expert axis
  constexpr int NPL = (BN + 31) / 32;           // logits per lane in the softmax
  constexpr int XS = TM * KC / 8;               // x slots of 8 k-values per chunk
  constexpr int WS = BN * KC / 4;               // W_r slots of 4 k-values per chunk
  constexpr int XPER = (XS + 31) / 32, WPER = (WS + 31) / 32;
  constexpr int STAGE = KC * (TM + BN);         // floats per warp buffer
  static_assert(TM * BN == 32 * 64, "one warp holds the whole tile");
  extern __shared__ __align__(16) float fsm[];
  __shared__ int eid[kTokensPerBlock];
  __shared__ int lead_count[kTokensPerBlock];
  __shared__ float s_psum[kWarps][BN];

  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    hdr->err = kDevOk;   // per-call device status
    hdr->done = 0u;      // arrival counter of the dispatch scan
  }
  const int t0 = blockIdx.x * TM;
  float* wbuf = fsm + warp * 2 * STAGE;         // this warp's two staging buffers
  const int tx = lane % TXN, ty = lane / TXN;
  const bool xvec = ((d * (int)sizeof(TX)) % 16 == 0) &&
                    ((reinterpret_cast<uintptr_t>(x) & 15) == 0);
  const bool wvec = ((d % 4) == 0) && ((reinterpret_cast<uintptr_t>(W_r) & 15) == 0);

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  float rx[XPER][8];
  float4 rw[WPER];
  auto gload = [&](int k0) {
#pragma unroll
    for (int q = 0; q < XPER; ++q) {
      const int sl = lane + 32 * q;
      if (sl < XS) {
        const int m = sl % TM, kq = sl / TM;
        const int t = t0 + m;
        if (t < T) {
          load8(x + (size_t)t * d, k0 + kq * 8, d, xvec, rx[q]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) rx[q][j] = 0.f;
        }
      }
    }
#pragma unroll
    for (int q = 0; q < WPER; ++q) {
      const int sl = lane + 32 * q;
      if (sl < WS) {
        const int n = sl % BN, kq = sl / BN;
        const int k = k0 + kq * 4;
        const float* wr = W_r + (size_t)n * d;
        if (n >= N) {
          rw[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else if (wvec && k + 4 <= d) {
          rw[q] = *reinterpret_cast<const float4*>(wr + k);
        } else {
          rw[q] = make_float4(k < d ? wr[k] : 0.f, k + 1 < d ? wr[k + 1] : 0.f,
                              k + 2 < d ? wr[k + 2] : 0.f, k + 3 < d ? wr[k + 3] : 0.f);
        }
      }
    }
  };
  auto sstore = [&](float* buf) {
    float* As = buf;              // [KC][TM]
    float* Bs = buf + KC * TM;    // [KC][BN]
#pragma unroll
    for (int q = 0; q < XPER; ++q) {
      const int sl = lane + 32 * q;
      if (sl < XS) {
        const int m = sl % TM, kq = sl / TM;
#pragma unroll
        for (int j = 0; j < 8; ++j) As[(kq * 8 + j) * TM + m] = rx[q][j];
      }
    }
#pragma unroll
    for (int q = 0; q < WPER; ++q) {
      const int sl = lane + 32 * q;
      if (sl < WS) {
        const int n = sl % BN, kq = sl / BN;
        Bs[(kq * 4 + 0) * BN + n] = rw[q].x;
        Bs[(kq * 4 + 1) * BN + n] = rw[q].y;
        Bs[(kq * 4 + 2) * BN + n] = rw[q].z;
        Bs[(kq * 4 + 3) * BN + n] = rw[q].w;
      }
    }
  };

  const int nchunks = (d + KC - 1) / KC;
  int buf = 0;
  if (warp < nchunks) {
    gload(warp * KC);
    sstore(wbuf);
    __syncwarp();
    for (int c = warp; c < nchunks; c += kWarps) {
      const bool more = c + kWarps < nchunks;
      if (more) gload((c + kWarps) * KC);
      const float* As = wbuf + buf * STAGE;
      const float* Bs = As + KC * TM;
#pragma unroll
      for (int k = 0; k < KC; ++k) {
        float a[8], b[8];
        *reinterpret_cast<float4*>(&a[0]) = *reinterpret_cast<const float4*>(&As[k * TM + ty * 8]);
        *reinterpret_cast<float4*>(&a[4]) =
            *reinterpret_cast<const float4*>(&As[k * TM + ty * 8 + 4]);
        *reinterpret_cast<float4*>(&b[0]) = *reinterpret_cast<const float4*>(&Bs[k * BN + tx * 4]);
        *reinterpret_cast<float4*>(&b[4]) =
            *reinterpret_cast<const float4*>(&Bs[k * BN + BN / 2 + tx * 4]);
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      if (more) {
        buf ^= 1;
        sstore(wbuf + buf * STAGE);
      }
      __syncwarp();
    }
  }
  __syncthreads();   // all warps are done with their staging buffers

  // partial tiles P[w][TM][BN] (aliases the staging area), summed in warp order
  float* P = fsm;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float* pr = P + (size_t)warp * TM * BN + (ty * 8 + i) * BN + tx * 4;
    *reinterpret_cast<float4*>(pr) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    *reinterpret_cast<float4*>(pr + BN / 2) =
        make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < TM * BN; idx += 256) {
    float v = P[idx];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) v += P[(size_t)w * TM * BN + idx];
    const int n = idx % BN;
    P[idx] = (n < N) ? v + (b_r ? b_r[n] : 0.f) : -INFINITY;   // in place: Z = P[0]
  }
  __syncthreads();

  // softmax, one warp per token
  const int ntok = max(0, min(TM, T - t0));
  float pacc[NPL];
#pragma unroll
  for (int j = 0; j < NPL; ++j) pacc[j] = 0.f;
  for (int i = warp; i < TM; i += kWarps) {
    if (i >= ntok) {
      if (lane == 0) eid[i] = -1;
      continue;
    }
    float v[NPL];
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const int n = lane + 32 * j;
      v[j] = (n < BN) ? P[i * BN + n] : -INFINITY;
    }
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
  for (int j = 0; j < NPL; ++j) {
    const int n = lane + 32 * j;
    if (n < BN) s_psum[warp][n] = pacc[j];
  }
  __syncthreads();
  block_ranks(eid, lead_count, ntok, TM, t0, local_rank);
  const int b = blockIdx.x;
  int* cnt_row = blk_count + (size_t)b * N;
  float* ps_row = blk_psum + (size_t)b * N;
  for (int n = threadIdx.x; n < N; n += 256) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) a += s_psum[w][n];
    ps_row[n] = a;
    cnt_row[n] = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ntok; i += 256) {
    if (lead_count[i] > 0) cnt_row[eid[i]] = lead_count[i];
  }
}

template <typename TX, int BN>
cudaError_t launch_warpsplit_t(const Shape& s, const Workspace& ws, const void* x, const float* W_r,
                           const float* b_r, int* expert_idx, float* gate, int* local_rank,
                           cudaStream_t stream) {
  constexpr int TM = 2048 / BN;
  constexpr int KC = BN <= 64 ? 16 : 8;
  const size_t stage_bytes = (size_t)8 * 2 * KC * (TM + BN) * sizeof(float);
  const size_t part_bytes = (size_t)8 * TM * BN * sizeof(float);
  const size_t smem = stage_bytes > part_bytes ? stage_bytes : part_bytes;
  cudaError_t e = cudaFuncSetAttribute(router_warpsplit_kernel<TX, BN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((s.T + TM - 1) / TM);
  router_warpsplit_kernel<TX, BN><<<grid, 256, smem, stream>>>(
      static_cast<const TX*>(x), W_r, b_r, (int)s.T, (int)s.d, (int)s.N, expert_idx, gate,
      local_rank, ws.blk_count, ws.blk_psum, ws.hdr);
  return cudaGetLastError();
}

// Big-tile router for large T and N <= BN: a cluster of S CTAs (S = 1 or 2,
// along z) owns BM tokens x BN experts; CTA r accumulates K slice r with 8 x 8
// register tiles (256 threads, main loop above) into its partial tile, then -
// after a cluster barrier - reduces rows [r*R, r*R+R) (R = BM/S) over the S
// partial tiles through distributed shared memory in rank order
// (deterministic), adds the bias and runs each token's softmax with one warp.
// Its R tokens form dispatch block tile*S + r.
template <typename TX, int BM, int BN>
__global__ void __launch_bounds__((BM / 8) * (BN / 8), 2)
router_tile_kernel(const TX* __restrict__ x, const float* __restrict__ W_r,
                   const float* __restrict__ b_r, int T, int d, int N, int kslice,
                   int* __restrict__ expert_idx, float* __restrict__ gate,
                   int* __restrict__ local_rank, int* __restrict__ blk_count,
                   float* __restrict__ blk_psum, WsHeader* hdr) {
  constexpr int kThreads = (BM / 8) * (BN / 8), kWarps = kThreads / 32;
  static_assert(kThreads == 256, "256 threads");
  constexpr int NPL = BN / 32;
  constexpr int PS = BN;                      // row stride of the partial tile
  constexpr int STAGE = 2 * kBK * (BM + BN);  // floats of the staging buffers
  extern __shared__ __align__(16) float fsm[];
  auto As = reinterpret_cast<float (*)[kBK][BM]>(fsm);                    // [2][kBK][BM]
  auto Bs = reinterpret_cast<float (*)[kBK][BN]>(fsm + 2 * kBK * BM);     // [2][kBK][BN]
  float* Ps = fsm + STAGE;                    // [BM][PS] this CTA's partial tile
  __shared__ float s_psum[kWarps][BN];
  __shared__ int eid[kTokensPerBlock];
  __shared__ int lead_count[kTokensPerBlock];
  cg::cluster_group cluster = cg::this_cluster();
  const int S = (int)cluster.num_blocks();
  const int r = (int)cluster.block_rank();
  pdl_trigger();
  pdl_wait();
  if (blockIdx.x == 0 && r == 0 && threadIdx.x == 0) {
    hdr->err = kDevOk;   // per-call device status
    hdr->done = 0u;      // arrival counter of the dispatch scan
  }
  const int tid = threadIdx.x;
  const int tx = tid % (BN / 8), ty = tid / (BN / 8);
  const int m0 = blockIdx.x * BM;
  const int k_lo = r * kslice;
  const int k_hi = min(d, k_lo + kslice);
  float acc[8][8];
  logits_mainloop<TX, BM, BN>(x, W_r, T, d, N, m0, 0, k_lo, k_hi, As, Bs, acc);
  // lane tx holds experts tx*4 + {0..3} and BN/2 + tx*4 + {0..3} (main loop layout)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float* pr = Ps + (ty * 8 + i) * PS + tx * 4;
    *reinterpret_cast<float4*>(pr) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    *reinterpret_cast<float4*>(pr + BN / 2) =
        make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
  }
  cluster.sync();   // every partial tile of the cluster is complete

  // Z: this CTA's R rows of logits + bias; in place in Ps when S == 1, else in
  // the (now free) staging area, which holds R x BN floats for R = BM/2.
  const int R = BM / S;
  const int row0 = r * R;
  float* Z = (S == 1) ? Ps : fsm;
  const int zs = (S == 1) ? PS : BN;
  const float* peer1 = cluster.map_shared_rank(Ps, S > 1 ? 1 : 0);
  const float* peer0 = cluster.map_shared_rank(Ps, 0);
  for (int idx = tid; idx < R * (BN / 4); idx += kThreads) {
    const int i = idx / (BN / 4), n = (idx % (BN / 4)) * 4;
    const int off = (row0 + i) * PS + n;
    float4 v = *reinterpret_cast<const float4*>(peer0 + off);
    if (S > 1) {
      const float4 u = *reinterpret_cast<const float4*>(peer1 + off);
      v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
    }
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int c = 0; c < 4; ++c)
      Z[i * zs + n + c] = (n + c < N) ? vv[c] + (b_r ? b_r[n + c] : 0.f) : -INFINITY;
  }
  __syncthreads();

  const int t0 = m0 + row0;
  const int ntok = max(0, min(R, T - t0));
  route_rows<NPL, kWarps>(Z, zs, R, ntok, t0, N, blockIdx.x * S + r, expert_idx, gate,
                          local_rank, blk_count, blk_psum, hdr, eid, lead_count, &s_psum[0][0]);
  cluster.sync();   // the peer has finished reading this CTA's partial tile
}

template <typename TX, int BM, int BN>
cudaError_t launch_tile_t(const Shape& s, const Workspace& ws, const void* x, const float* W_r,
                          const float* b_r, int* expert_idx, float* gate, int* local_rank,
                          cudaStream_t stream) {
  const size_t smem = ((size_t)2 * kBK * (BM + BN) + (size_t)BM * BN) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(router_tile_kernel<TX, BM, BN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((s.T + BM - 1) / BM), 1, (unsigned)s.ksplit_eff);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)s.ksplit_eff;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, router_tile_kernel<TX, BM, BN>, static_cast<const TX*>(x), W_r,
                            b_r, (int)s.T, (int)s.d, (int)s.N, s.kslice, expert_idx, gate,
                            local_rank, ws.blk_count, ws.blk_psum, ws.hdr);
}

template <typename TX, int BM, int BN>
cudaError_t launch_logits_t(const Shape& s, const Workspace& ws, const void* x, const float* W_r,
                            cudaStream_t stream) {
  const int T = (int)s.T, d = (int)s.d, N = (int)s.N;
  const int kslice = s.kslice;
  const int nz = s.ksplit_eff;
  dim3 grid((T + BM - 1) / BM, (N + BN - 1) / BN, nz);
  router_logits_kernel<TX, BM, BN><<<grid, (BM / 8) * (BN / 8), 0, stream>>>(
      static_cast<const TX*>(x), W_r, ws.logits, T, d, N, kslice, ws.hdr);
  return cudaGetLastError();
}

template <int NPL>
cudaError_t launch_softmax_t(const Shape& s, const Workspace& ws, const float* b_r,
                             int* expert_idx, float* gate, int* local_rank, cudaStream_t stream) {
  const size_t smem = (size_t)(kSoftmaxWarps + 1) * s.N * sizeof(float);
  auto kern = s.topk == 2 ? router_softmax_kernel<NPL, true> : router_softmax_kernel<NPL, false>;
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_dependent(kern, dim3(s.nblk), dim3(kSoftmaxThreads), smem, stream,
                          static_cast<const float*>(ws.logits), s.ksplit_eff, b_r, (int)s.T,
                          (int)s.N, s.tpb, expert_idx, gate, local_rank, ws.blk_count,
                          ws.blk_psum, ws.blk_count1, s.normalize, ws.hdr);
}

}  // namespace

RouterPlan router_plan(int64_t T, int64_t d, int64_t N, int tensor, int topk, int force_wide) {
  RouterPlan p;
  // force_wide (tensor cores only): the logits GEMM and a separate softmax at any
  // N, for a jittered input, which only that logits kernel takes as bf16 pieces
  if (!tensor) force_wide = 0;
  if (tensor && N <= kFusedRouterMaxN && topk == 1 && !force_wide) {
    // tensor cores: 128-token tiles; K split over 2 or 4 CTAs of a cluster while
    // the tiles alone would leave most SMs idle (and each CTA keeps >= 2 k-blocks)
    const int64_t tiles = (T + 127) / 128;
    const int64_t nkb = (d + 63) / 64;
    int64_t S = 1;
    while (S < 4 && tiles * S * 2 <= 160 && 2 * S * 2 <= nkb) S *= 2;
    const int64_t kb_per = (nkb + S - 1) / S;
    p.path = kRouterTC;
    p.ksplit = (int)S;
    p.kslice = (int)(kb_per * 64);
    p.tpb = (int)(128 / S);
    return p;
  }
  if (N <= kFusedRouterMaxN && topk == 1 && !force_wide) {
    // one fused kernel; big tiles once there are enough of them to fill the GPU
    const int64_t bm = N <= 64 ? 256 : 128;
    const int64_t tiles = (T + bm - 1) / bm;
    if (N > 32 && tiles >= 100) {
      // two K slices over a 2-CTA cluster until there are ~2 CTAs per SM
      p.path = kRouterTile;
      p.ksplit = (tiles < 2 * 148 && d >= 128) ? 2 : 1;
      p.kslice = (int)(((d + p.ksplit - 1) / p.ksplit + kBK - 1) / kBK * kBK);
      p.ksplit = (int)((d + p.kslice - 1) / p.kslice);
      p.tpb = (int)(bm / p.ksplit);
    } else {
      p.path = kRouterWarpSplit;
      p.tpb = N <= 32 ? 64 : (N <= 64 ? 32 : 16);
      p.kslice = (int)((d + kBK - 1) / kBK * kBK);
      p.ksplit = 1;
    }
    return p;
  }
  // wide N (and every top-2 layer): logits GEMM in 128 x 128 tiles (bf16
  // layers: tensor cores over the whole K; fp32 layers: FFMA with K slices for
  // ~3 CTAs per SM), then the softmax kernel over blocks of 128/64/32 tokens
  p.tpb = 32;
  for (int tpb = 128; tpb > 32; tpb /= 2)
    if ((T + tpb - 1) / tpb >= 2 * 148) { p.tpb = tpb; break; }
  if (tensor && N % 4 == 0 && N <= kStreamSoftmaxMaxN) {
    // the streaming softmax's persistent CTAs (one per SM) take whole blocks:
    // blocks of up to 128 tokens sized so that every CTA gets the same number
    const int64_t rounds = (T + 128 * 148 - 1) / (128 * 148);
    const int64_t tpb = (T + rounds * 148 - 1) / (rounds * 148);
    p.tpb = static_cast<int>(tpb < 32 ? 32 : tpb);
  }
  if (tensor) {
    p.path = kRouterTCWide;
    p.ksplit = 1;
    p.kslice = (int)((d + 63) / 64 * 64);
    return p;
  }
  p.path = kRouterWide;
  int64_t tiles = ((T + 127) / 128) * ((N + 127) / 128);
  if (tiles < 1) tiles = 1;
  int64_t ks = (3 * 148 + tiles - 1) / tiles;
  const int64_t max_ks = d / 64 > 0 ? d / 64 : 1;
  if (ks > max_ks) ks = max_ks;
  if (ks > 16) ks = 16;
  if (ks < 1) ks = 1;
  p.kslice = (int)(((d + ks - 1) / ks + kBK - 1) / kBK * kBK);
  p.ksplit = (int)((d + p.kslice - 1) / p.kslice);
  p.tpb = 32;
  for (int tpb = 128; tpb > 32; tpb /= 2)
    if ((T + tpb - 1) / tpb >= 2 * 148) { p.tpb = tpb; break; }
  return p;
}

template <typename TX>
__global__ void __launch_bounds__(256)
router_jitter_kernel(const TX* __restrict__ x, const float* __restrict__ noise,
                     float* __restrict__ xj, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    xj[i] = static_cast<float>(x[i]) * noise[i];
}

// The jittered input for the tensor-core logits: v = x * noise in fp32, split
// exactly into three bf16 numbers v = hi + mid + lo (each residual is exact in
// fp32, and 3 x 8 significand bits cover fp32's 24), stored as the pieces
// [hi; mid; lo] of a bf16 [3T, d] matrix.
__global__ void __launch_bounds__(256)
router_jitter_split_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ noise,
                           __nv_bfloat16* __restrict__ x3, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const float v = __bfloat162float(x[i]) * noise[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(m);
    x3[i] = h;
    x3[n + i] = m;
    x3[2 * n + i] = __float2bfloat16_rn(r2);
  }
}

cudaError_t launch_router_jitter(const Shape& s, const Workspace& ws, const void* x,
                                 const float* noise, cudaStream_t stream) {
  const size_t n = static_cast<size_t>(s.T) * static_cast<size_t>(s.d);
  size_t blocks = (n + 255) / 256;
  if (blocks > 8 * 148) blocks = 8 * 148;
  if (blocks < 1) blocks = 1;
  if (s.xsplit)
    router_jitter_split_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), noise, static_cast<__nv_bfloat16*>(ws.x3), n);
  else if (s.dtype == 1)
    router_jitter_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), noise, ws.xj, n);
  else
    router_jitter_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const float*>(x), noise, ws.xj, n);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_router_logits(const Shape& s, const Workspace& ws, const void* x,
                                 const float* W_r, const float* b_r, int* expert_idx, float* gate,
                                 int* local_rank, cudaStream_t stream) {
  cudaError_t e;
  const bool bf = s.dtype == 1 && !s.jitter;   // a jittered input is fp32
  if (s.router_path == kRouterTile) {
    if (s.N <= 64)
      e = bf ? launch_tile_t<__nv_bfloat16, 256, 64>(s, ws, x, W_r, b_r, expert_idx, gate,
                                                      local_rank, stream)
             : launch_tile_t<float, 256, 64>(s, ws, x, W_r, b_r, expert_idx, gate, local_rank,
                                              stream);
    else
      e = bf ? launch_tile_t<__nv_bfloat16, 128, 128>(s, ws, x, W_r, b_r, expert_idx, gate,
                                                       local_rank, stream)
             : launch_tile_t<float, 128, 128>(s, ws, x, W_r, b_r, expert_idx, gate, local_rank,
                                               stream);
  } else if (s.router_path == kRouterWarpSplit) {
    if (s.N <= 32)
      e = bf ? launch_warpsplit_t<__nv_bfloat16, 32>(s, ws, x, W_r, b_r, expert_idx, gate,
                                                      local_rank, stream)
             : launch_warpsplit_t<float, 32>(s, ws, x, W_r, b_r, expert_idx, gate, local_rank,
                                              stream);
    else if (s.N <= 64)
      e = bf ? launch_warpsplit_t<__nv_bfloat16, 64>(s, ws, x, W_r, b_r, expert_idx, gate,
                                                      local_rank, stream)
             : launch_warpsplit_t<float, 64>(s, ws, x, W_r, b_r, expert_idx, gate, local_rank,
                                              stream);
    else
      e = bf ? launch_warpsplit_t<__nv_bfloat16, 128>(s, ws, x, W_r, b_r, expert_idx, gate,
                                                       local_rank, stream)
             : launch_warpsplit_t<float, 128>(s, ws, x, W_r, b_r, expert_idx, gate, local_rank,
                                               stream);
  } else {
    e = bf ? launch_logits_t<__nv_bfloat16, 128, 128>(s, ws, x, W_r, stream)
           : launch_logits_t<float, 128, 128>(s, ws, x, W_r, stream);
  }
  count_launch();
  return e;
}

int softmax_variant(const Shape& s) {
  if (s.router_path != kRouterWide && s.router_path != kRouterTCWide) return kSoftmaxFused;
  if (s.ksplit_eff == 1 && s.N % 4 == 0 && s.N <= kStreamSoftmaxMaxN) return kSoftmaxStream;
  return (s.N + 31) / 32 <= 64 ? kSoftmaxRows : kSoftmaxWide;
}

template <int V4, int WPR>
cudaError_t launch_stream_t(const Shape& s, const Workspace& ws, const float* b_r,
                            int* expert_idx, float* gate, int* local_rank, cudaStream_t stream) {
  const size_t smem = stream_softmax_smem(static_cast<int>(s.N));
  const bool full = s.N == 128 * WPR * V4;
  auto kern = s.topk == 2 ? router_softmax_stream_kernel<V4, WPR, true, false>
                          : (full ? router_softmax_stream_kernel<V4, WPR, false, true>
                                  : router_softmax_stream_kernel<V4, WPR, false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int grid = s.nblk < sms ? s.nblk : sms;
  return launch_dependent(kern, dim3(grid), dim3(kStreamThreads), smem, stream,
                          static_cast<const float*>(ws.logits), b_r, (int)s.T, (int)s.N, s.tpb,
                          s.nblk, expert_idx, gate, local_rank, ws.blk_count, ws.blk_psum,
                          ws.blk_count1, s.normalize, ws.hdr, wait_limit_ns());
}

cudaError_t launch_router_softmax(const Shape& s, const Workspace& ws, const float* b_r,
                                  int* expert_idx, float* gate, int* local_rank,
                                  cudaStream_t stream) {
  cudaError_t e;
  const int64_t npl = (s.N + 31) / 32;
  if (softmax_variant(s) == kSoftmaxStream) {
    // float4 columns per lane: a row (N <= 1024) or half a row (N <= 2048) per warp
    const int wpr = stream_wpr(static_cast<int>(s.N));
    const int64_t v4 = ((s.N / 4 + wpr - 1) / wpr + 31) / 32;
    if (wpr == 2) e = launch_stream_t<8, 2>(s, ws, b_r, expert_idx, gate, local_rank, stream);
    else if (v4 <= 1) e = launch_stream_t<1, 1>(s, ws, b_r, expert_idx, gate, local_rank, stream);
    else if (v4 <= 2) e = launch_stream_t<2, 1>(s, ws, b_r, expert_idx, gate, local_rank, stream);
    else if (v4 <= 4) e = launch_stream_t<4, 1>(s, ws, b_r, expert_idx, gate, local_rank, stream);
    else e = launch_stream_t<8, 1>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  } else if (npl <= 1) e = launch_softmax_t<1>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 2) e = launch_softmax_t<2>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 4) e = launch_softmax_t<4>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 8) e = launch_softmax_t<8>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 16) e = launch_softmax_t<16>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 32) e = launch_softmax_t<32>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 64) e = launch_softmax_t<64>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else {
    e = launch_dependent(router_softmax_wide_kernel, dim3(s.nblk), dim3(kSoftmaxThreads), 0,
                         stream, ws.logits, s.ksplit_eff, b_r, (int)s.T, (int)s.N, s.tpb,
                         expert_idx, gate, local_rank, ws.blk_count, ws.blk_psum, ws.hdr);
  }
  count_launch();
  return e;
}

}  // namespace swl
