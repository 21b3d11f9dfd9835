// Router of the Switch layer, in fp32 ("selective precision": the router input
// is cast to float32 and logits, softmax and the argmax are computed in fp32;
// paper-graph summary of arXiv 2101.03961, section 3.4 "The selective precision
// solution"; Switch Transformer, explained, recipe step 2).
//
//   logits  z_t = W_r x_t (+ b_r)            "The mathematics of routing": h(x) = W_r x
//   probs   p_t = softmax(z_t)                p_i = exp(h_i) / sum_j exp(h_j)
//   choice  e_t = argmax_i p_t,i (lowest index on ties), gate g_t = p_t,e_t
//
// Stage 1 (router_logits_kernel): register-tiled fp32 FFMA GEMM [T,d] x [N,d]^T.
// Stage 2 (router_softmax_kernel): one CTA per block of 128 tokens; one warp per
//   token row for max/argmax/sum via warp shuffles; then, per block, the
//   in-block rank of every token among the block's tokens with the same expert,
//   the block's per-expert token counts, and per-expert sums of p (token order).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace swl {
namespace {

constexpr int kLogitsThreads = 256;
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

// z[t, n] = sum_k x[t, k] * W_r[n, k] + b_r[n].  CTA tile BM tokens x BN experts,
// 256 threads, 8 x 8 outputs per thread, K staged through shared memory in
// chunks of 16 with register prefetch of the next chunk.
template <typename TX, int BM, int BN>
__global__ void __launch_bounds__(kLogitsThreads)
router_logits_kernel(const TX* __restrict__ x, const float* __restrict__ W_r,
                     const float* __restrict__ b_r, float* __restrict__ z, int T, int d, int N,
                     WsHeader* hdr) {
  static_assert((BM / 8) * (BN / 8) == kLogitsThreads, "thread tile");
  __shared__ __align__(16) float As[2][kBK][BM];
  __shared__ __align__(16) float Bs[2][kBK][BN];

  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    hdr->err = kDevOk;   // per-call device status
    hdr->done = 0u;      // arrival counter of the dispatch scan
  }

  const int tid = threadIdx.x;
  const int tx = tid % (BN / 8);
  const int ty = tid / (BN / 8);
  const int m0 = blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  const bool xvec = ((d * (int)sizeof(TX)) % 16 == 0) &&
                    ((reinterpret_cast<uintptr_t>(x) & 15) == 0);
  const bool wvec = ((d % 4) == 0) && ((reinterpret_cast<uintptr_t>(W_r) & 15) == 0);

  constexpr int A_SLOTS = BM * 2;   // (token, k-half) pairs per chunk
  constexpr int B_SLOTS = BN * 2;
  constexpr int A_PER = (A_SLOTS + kLogitsThreads - 1) / kLogitsThreads;
  constexpr int B_PER = (B_SLOTS + kLogitsThreads - 1) / kLogitsThreads;
  float ra[A_PER][8];
  float rb[B_PER][8];

  auto gload = [&](int k0) {
#pragma unroll
    for (int i = 0; i < A_PER; ++i) {
      const int s = tid + i * kLogitsThreads;
      if (s < A_SLOTS) {
        const int m = s % BM, kh = s / BM;
        const int t = m0 + m;
        if (t < T) {
          load8(x + (size_t)t * d, k0 + kh * 8, d, xvec, ra[i]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) ra[i][j] = 0.f;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < B_PER; ++i) {
      const int s = tid + i * kLogitsThreads;
      if (s < B_SLOTS) {
        const int n = s % BN, kh = s / BN;
        if (n0 + n < N) {
          load8(W_r + (size_t)(n0 + n) * d, k0 + kh * 8, d, wvec, rb[i]);
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
      const int s = tid + i * kLogitsThreads;
      if (s < A_SLOTS) {
        const int m = s % BM, kh = s / BM;
#pragma unroll
        for (int j = 0; j < 8; ++j) As[buf][kh * 8 + j][m] = ra[i][j];
      }
    }
#pragma unroll
    for (int i = 0; i < B_PER; ++i) {
      const int s = tid + i * kLogitsThreads;
      if (s < B_SLOTS) {
        const int n = s % BN, kh = s / BN;
#pragma unroll
        for (int j = 0; j < 8; ++j) Bs[buf][kh * 8 + j][n] = rb[i][j];
      }
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int nk = (d + kBK - 1) / kBK;
  gload(0);
  sstore(0);
  __syncthreads();
  for (int kc = 0; kc < nk; ++kc) {
    const int buf = kc & 1;
    if (kc + 1 < nk) gload((kc + 1) * kBK);
#pragma unroll
    for (int k = 0; k < kBK; ++k) {
      float a[8], b[8];
      *reinterpret_cast<float4*>(&a[0]) = *reinterpret_cast<const float4*>(&As[buf][k][ty * 8]);
      *reinterpret_cast<float4*>(&a[4]) =
          *reinterpret_cast<const float4*>(&As[buf][k][ty * 8 + 4]);
      *reinterpret_cast<float4*>(&b[0]) = *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 8]);
      *reinterpret_cast<float4*>(&b[4]) =
          *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 8 + 4]);
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (kc + 1 < nk) sstore(buf ^ 1);
    __syncthreads();
  }

  float bias[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int n = n0 + tx * 8 + j;
    bias[j] = (b_r != nullptr && n < N) ? b_r[n] : 0.f;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = m0 + ty * 8 + i;
    if (t >= T) continue;
    float* zr = z + (size_t)t * N;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + tx * 8 + j;
      if (n < N) zr[n] = acc[i][j] + bias[j];
    }
  }
}

constexpr int kSoftmaxThreads = 256;
constexpr int kSoftmaxWarps = kSoftmaxThreads / 32;

// One CTA per block of kTokensPerBlock tokens.
//  * per token (one warp): m = max_i z_i with its lowest index, s = sum exp(z_i - m),
//    gate = p at the argmax = 1/s; the row of z is overwritten with p_i = exp(z_i - m)/s.
//  * per block: in-block rank of each token among earlier tokens with the same
//    expert (stored in local_rank), per-expert token count blk_count[b][e], and
//    per-expert probability sum blk_psum[b][e] summed in token order.
__global__ void __launch_bounds__(kSoftmaxThreads)
router_softmax_kernel(float* __restrict__ zp, int T, int N, int* __restrict__ expert_idx,
                      float* __restrict__ gate, int* __restrict__ local_rank,
                      int* __restrict__ blk_count, float* __restrict__ blk_psum,
                      WsHeader* hdr) {
  __shared__ int eid[kTokensPerBlock];
  __shared__ int lead_count[kTokensPerBlock];
  const int b = blockIdx.x;
  const int t0 = b * kTokensPerBlock;
  const int ntok = min(kTokensPerBlock, T - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = warp; i < kTokensPerBlock; i += kSoftmaxWarps) {
    if (i >= ntok) {
      if (lane == 0) eid[i] = -1;
      continue;
    }
    const int t = t0 + i;
    float* row = zp + (size_t)t * N;
    float best = -INFINITY;
    int bidx = 0x7fffffff;
    for (int j = lane; j < N; j += 32) {
      const float v = row[j];
      if (v > best) { best = v; bidx = j; }   // strict: keeps the first index within a lane
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
      if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
    }
    float s = 0.f;
    for (int j = lane; j < N; j += 32) {
      const float e = expf(row[j] - best);
      row[j] = e;
      s += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float inv = 1.0f / s;
    for (int j = lane; j < N; j += 32) row[j] *= inv;
    if (bidx >= N) {          // no finite maximum (non-finite logits): flag, keep in range
      bidx = 0;
      if (lane == 0) atomicExch(&hdr->err, kDevNonFiniteLogits);
    }
    if (lane == 0) {
      expert_idx[t] = bidx;
      gate[t] = inv;            // p at the argmax: exp(0) / s
      eid[i] = bidx;
    }
  }
  __syncthreads();

  // in-block stable rank and per-expert counts (leaders = first token of an expert)
  for (int i = threadIdx.x; i < kTokensPerBlock; i += kSoftmaxThreads) {
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
  // per-expert column sums of p over the block (token order), zero counts
  int* cnt_row = blk_count + (size_t)b * N;
  float* ps_row = blk_psum + (size_t)b * N;
  for (int e = threadIdx.x; e < N; e += kSoftmaxThreads) {
    float acc = 0.f;
    const float* col = zp + (size_t)t0 * N + e;
    for (int i = 0; i < ntok; ++i) acc += col[(size_t)i * N];
    ps_row[e] = acc;
    cnt_row[e] = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ntok; i += kSoftmaxThreads) {
    if (lead_count[i] > 0) cnt_row[eid[i]] = lead_count[i];
  }
}

}  // namespace

// Wide expert tiles when N is large, tall token tiles when N is small.
cudaError_t launch_router_logits(const Shape& s, const Workspace& ws, const void* x,
                                 const float* W_r, const float* b_r, cudaStream_t stream) {
  float* logits = ws.logits;
  WsHeader* hdr = ws.hdr;
  const int T = (int)s.T, d = (int)s.d, N = (int)s.N;
  if (N > 64) {
    constexpr int BM = 128, BN = 128;
    dim3 grid((T + BM - 1) / BM, (N + BN - 1) / BN);
    if (s.dtype == 1)
      router_logits_kernel<__nv_bfloat16, BM, BN><<<grid, kLogitsThreads, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(x), W_r, b_r, logits, T, d, N, hdr);
    else
      router_logits_kernel<float, BM, BN><<<grid, kLogitsThreads, 0, stream>>>(
          static_cast<const float*>(x), W_r, b_r, logits, T, d, N, hdr);
  } else {
    constexpr int BM = 256, BN = 64;
    dim3 grid((T + BM - 1) / BM, (N + BN - 1) / BN);
    if (s.dtype == 1)
      router_logits_kernel<__nv_bfloat16, BM, BN><<<grid, kLogitsThreads, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(x), W_r, b_r, logits, T, d, N, hdr);
    else
      router_logits_kernel<float, BM, BN><<<grid, kLogitsThreads, 0, stream>>>(
          static_cast<const float*>(x), W_r, b_r, logits, T, d, N, hdr);
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_router_softmax(const Shape& s, const Workspace& ws, int* expert_idx,
                                  float* gate, int* local_rank, cudaStream_t stream) {
  router_softmax_kernel<<<s.nblk, kSoftmaxThreads, 0, stream>>>(
      ws.logits, (int)s.T, (int)s.N, expert_idx, gate, local_rank, ws.blk_count, ws.blk_psum, ws.hdr);
  count_launch();
  return cudaGetLastError();
}

}  // namespace swl
