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
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

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

// Partial logits over one K slice: zpart[ks][t][n] = sum_{k in slice ks} x[t,k] W_r[n,k].
// CTA tile BM tokens x BN experts, (BM/8)*(BN/8) threads with 8 x 8 outputs each,
// K staged through shared memory in chunks of 16 with register prefetch of the
// next chunk.  Splitting K (blockIdx.z) gives enough CTAs to fill the GPU when T
// and N are small; the softmax kernel adds the slices in order, then the bias.
template <typename TX, int BM, int BN>
__global__ void __launch_bounds__((BM / 8) * (BN / 8))
router_logits_kernel(const TX* __restrict__ x, const float* __restrict__ W_r,
                     float* __restrict__ zpart, int T, int d, int N, int kslice,
                     WsHeader* hdr) {
  constexpr int kThreads = (BM / 8) * (BN / 8);
  __shared__ __align__(16) float As[2][kBK][BM];
  __shared__ __align__(16) float Bs[2][kBK][BN];

  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) {
    hdr->err = kDevOk;   // per-call device status
    hdr->done = 0u;      // arrival counter of the dispatch scan
  }

  const int tid = threadIdx.x;
  const int tx = tid % (BN / 8);
  const int ty = tid / (BN / 8);
  const int m0 = blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  const int k_lo = blockIdx.z * kslice;
  const int k_hi = min(d, k_lo + kslice);
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

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int nk = (k_hi - k_lo + kBK - 1) / kBK;
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

  float* zs = zpart + (size_t)blockIdx.z * T * N;
  const bool vec_out = (N % 4) == 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = m0 + ty * 8 + i;
    if (t >= T) continue;
    float* zr = zs + (size_t)t * N + n0 + tx * 8;
    if (vec_out && n0 + tx * 8 + 8 <= N) {
      *reinterpret_cast<float4*>(zr) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      *reinterpret_cast<float4*>(zr + 4) =
          make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (n0 + tx * 8 + j < N) zr[j] = acc[i][j];
    }
  }
}

constexpr int kSoftmaxThreads = 256;
constexpr int kSoftmaxWarps = kSoftmaxThreads / 32;

// Block-level bookkeeping shared by both softmax kernels: in-block stable rank
// of each token among the block's earlier tokens with the same expert, and the
// block's per-expert token counts (written by the first token of each expert).
// eid[i] < 0 marks an absent token.  Caller zeroes cnt_row before calling and
// synchronises the block after.
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

// One CTA per block of tpb tokens; one warp per token with the row of logits
// held in registers (NPL = logits per lane, N <= 32*NPL):
//   z = sum of the K-slice partials + b_r; m = max with the lowest index;
//   s = sum exp(z - m); gate = p at the argmax = 1/s; p_i = exp(z_i - m)/s is
//   accumulated per lane into per-expert sums.
// Then per block: ranks, counts blk_count[b][e], probability sums blk_psum[b][e]
// (each warp's tokens in order, warps in order).
template <int NPL>
__global__ void __launch_bounds__(kSoftmaxThreads)
router_softmax_kernel(const float* __restrict__ zpart, int nsplit, const float* __restrict__ b_r,
                      int T, int N, int tpb, int* __restrict__ expert_idx,
                      float* __restrict__ gate, int* __restrict__ local_rank,
                      int* __restrict__ blk_count, float* __restrict__ blk_psum,
                      WsHeader* hdr) {
  extern __shared__ float smem_f[];
  float* s_bias = smem_f;                 // [N]
  float* s_psum = smem_f + N;             // [kSoftmaxWarps][N]
  __shared__ int eid[kTokensPerBlock];
  __shared__ int lead_count[kTokensPerBlock];
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
      if (lane == 0) eid[i] = -1;
      continue;
    }
    const int t = t0 + i;
    const float* row = zpart + (size_t)t * N;
    float v[NPL];
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const int n = lane + 32 * j;
      if (n < N) {
        float a = row[n];
        for (int s = 1; s < nsplit; ++s) a += row[s * slice + n];
        v[j] = a + s_bias[n];
      } else {
        v[j] = -INFINITY;
      }
    }
    float best = -INFINITY;
    int bidx = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NPL; ++j)
      if (v[j] > best) { best = v[j]; bidx = lane + 32 * j; }   // first index within a lane
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
    for (int j = 0; j < NPL; ++j) acc[j] += v[j] * inv;
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
#pragma unroll
  for (int j = 0; j < NPL; ++j) {
    const int n = lane + 32 * j;
    if (n < N) s_psum[warp * N + n] = acc[j];
  }
  __syncthreads();
  block_ranks(eid, lead_count, ntok, tpb, t0, local_rank);
  int* cnt_row = blk_count + (size_t)b * N;
  float* ps_row = blk_psum + (size_t)b * N;
  for (int n = threadIdx.x; n < N; n += kSoftmaxThreads) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kSoftmaxWarps; ++w) a += s_psum[w * N + n];
    ps_row[n] = a;
    cnt_row[n] = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ntok; i += kSoftmaxThreads) {
    if (lead_count[i] > 0) cnt_row[eid[i]] = lead_count[i];
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
    if (bidx >= N) {
      bidx = 0;
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
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(
        router_softmax_kernel<NPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  router_softmax_kernel<NPL><<<s.nblk, kSoftmaxThreads, smem, stream>>>(
      ws.logits, s.ksplit_eff, b_r, (int)s.T, (int)s.N, s.tpb, expert_idx, gate, local_rank,
      ws.blk_count, ws.blk_psum, ws.hdr);
  return cudaGetLastError();
}

}  // namespace

int router_kslice(int64_t T, int64_t d, int64_t N) {
  // CTAs of the logits kernel before splitting K; aim for ~3 per SM on 148 SMs
  int64_t tiles = N > 64 ? ((T + 127) / 128) * ((N + 127) / 128)
                         : ((T + 127) / 128) * ((N + 63) / 64);
  if (tiles < 1) tiles = 1;   // empty batch
  int64_t ks = (3 * 148 + tiles - 1) / tiles;
  const int64_t max_ks = d / 64 > 0 ? d / 64 : 1;   // each slice keeps >= 64 of K
  if (ks > max_ks) ks = max_ks;
  if (ks > 16) ks = 16;
  if (ks < 1) ks = 1;
  return (int)(((d + ks - 1) / ks + kBK - 1) / kBK * kBK);
}

cudaError_t launch_router_logits(const Shape& s, const Workspace& ws, const void* x,
                                 const float* W_r, const float* b_r, cudaStream_t stream) {
  (void)b_r;   // the bias is added by the softmax kernel after the K slices
  cudaError_t e;
  if (s.N > 64) {
    e = s.dtype == 1 ? launch_logits_t<__nv_bfloat16, 128, 128>(s, ws, x, W_r, stream)
                     : launch_logits_t<float, 128, 128>(s, ws, x, W_r, stream);
  } else {
    e = s.dtype == 1 ? launch_logits_t<__nv_bfloat16, 128, 64>(s, ws, x, W_r, stream)
                     : launch_logits_t<float, 128, 64>(s, ws, x, W_r, stream);
  }
  count_launch();
  return e;
}

cudaError_t launch_router_softmax(const Shape& s, const Workspace& ws, const float* b_r,
                                  int* expert_idx, float* gate, int* local_rank,
                                  cudaStream_t stream) {
  cudaError_t e;
  const int64_t npl = (s.N + 31) / 32;
  if (npl <= 1) e = launch_softmax_t<1>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 2) e = launch_softmax_t<2>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 4) e = launch_softmax_t<4>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 8) e = launch_softmax_t<8>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 16) e = launch_softmax_t<16>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 32) e = launch_softmax_t<32>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else if (npl <= 64) e = launch_softmax_t<64>(s, ws, b_r, expert_idx, gate, local_rank, stream);
  else {
    router_softmax_wide_kernel<<<s.nblk, kSoftmaxThreads, 0, stream>>>(
        ws.logits, s.ksplit_eff, b_r, (int)s.T, (int)s.N, s.tpb, expert_idx, gate, local_rank,
        ws.blk_count, ws.blk_psum, ws.hdr);
    e = cudaGetLastError();
  }
  count_launch();
  return e;
}

}  // namespace swl
