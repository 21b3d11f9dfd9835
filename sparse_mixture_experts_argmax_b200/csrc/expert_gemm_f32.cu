// fp32 expert FFN GEMMs (CUDA cores, FFMA) for layers whose activations and
// expert weights are fp32.  Same packed-row layout and fused epilogues as the
// bf16 tensor-core path:
//   GEMM1: hbuf[r, :]  = relu(W1[e] xbuf[r, :] + b1[e])
//   GEMM2: out[tok, :] = g_tok * (W2[e] hbuf[r, :] + b2[e]),  tok = slot_token[r]
// (Switch Transformer reading note, "Expert FFN Layer" and "Router").
// Tensor cores are not used here: tf32 would not meet a 1e-4 tolerance.
//
// CTA = 32 output features x 32 packed rows of one expert; 256 threads, 4
// outputs each; K staged through shared memory in chunks of 32.  grid.x walks
// the per-expert row tiles through the device tile prefix (tile rows = 32),
// grid.y the 32-feature blocks.
#include <cuda_runtime.h>

#include "kernels.h"

namespace swl {
namespace {

constexpr int kTile = kF32TileRows;   // 32

// GLU (GEMM1 of GEGLU experts): W is [N, 2M, K], gate rows then value rows;
// out = GELU(gate + b_g) * (value + b_v) with the biases [N, 2M] laid out the same.
template <bool GLU>
__global__ void __launch_bounds__(256)
expert_gemm_f32_kernel(const float* __restrict__ act, const float* __restrict__ W,
                       const float* __restrict__ bias, const int* __restrict__ tile_prefix,
                       const int* __restrict__ exp_rows, const int* __restrict__ exp_base,
                       const int* __restrict__ slot_token, const float* __restrict__ gate,
                       float* __restrict__ out, int num_experts, int M, int K, int mode,
                       int T_rows, int* err) {
  __shared__ float As[kTile][kTile + 1];   // [row][k]
  __shared__ float Ws[kTile][kTile + 1];   // [feature][k]
  __shared__ float Wv[GLU ? kTile : 1][kTile + 1];   // value rows (GLU)
  pdl_trigger();
  pdl_wait();   // packed rows and tile prefix come from the dispatch
  const int g = blockIdx.x;
  if (g >= tile_prefix[num_experts]) return;
  int lo = 0, hi = num_experts;            // last e with prefix[e] <= g
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_prefix[mid] <= g) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int nt = g - tile_prefix[e];
  const int r0 = exp_base[e] + nt * kTile;
  const int nrows = min(kTile, exp_rows[e] - nt * kTile);
  const int m0 = blockIdx.y * kTile;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // feature, row group
  const int rows_e = GLU ? 2 * M : M;       // weight rows (and biases) per expert
  const float* We = W + (size_t)e * rows_e * K;

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float accv[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < K; k0 += kTile) {
    for (int i = threadIdx.x; i < kTile * kTile; i += 256) {
      const int rr = i / kTile, kk = i % kTile;
      As[rr][kk] = (rr < nrows && k0 + kk < K) ? act[(size_t)(r0 + rr) * K + k0 + kk] : 0.f;
      Ws[rr][kk] = (m0 + rr < M && k0 + kk < K) ? We[(size_t)(m0 + rr) * K + k0 + kk] : 0.f;
      if (GLU)
        Wv[rr][kk] = (m0 + rr < M && k0 + kk < K) ? We[(size_t)(M + m0 + rr) * K + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kTile; ++kk) {
      const float w = Ws[tx][kk];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(As[ty * 4 + i][kk], w, acc[i]);
      if (GLU) {
        const float wv = Wv[tx][kk];
#pragma unroll
        for (int i = 0; i < 4; ++i) accv[i] = fmaf(As[ty * 4 + i][kk], wv, accv[i]);
      }
    }
    __syncthreads();
  }
  const int m = m0 + tx;
  if (m >= M) return;
  const float bm = bias[(size_t)e * rows_e + m];
  if constexpr (GLU) {
    const float bv = bias[(size_t)e * rows_e + M + m];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = ty * 4 + i;
      if (rr >= nrows) continue;
      if (!checked_index(r0 + rr >= 0 && r0 + rr < T_rows, err)) continue;
      const float g = acc[i] + bm;
      out[(size_t)(r0 + rr) * M + m] = 0.5f * g * (1.0f + erff(g * 0.70710678118654752f)) *
                                       (accv[i] + bv);
    }
    return;
  } else {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = ty * 4 + i;
    if (rr >= nrows) continue;
    if (!checked_index(r0 + rr >= 0 && r0 + rr < T_rows, err)) continue;
    const float v = acc[i] + bm;
    if (mode == 0) {
      out[(size_t)(r0 + rr) * M + m] = fmaxf(v, 0.f);
    } else if (mode == 2) {        // packed rows without the gate (expert-parallel)
      out[(size_t)(r0 + rr) * M + m] = v;
    } else {
      const int tok = slot_token[r0 + rr];
      if (!checked_index(tok >= 0 && tok < T_rows, err)) continue;
      out[(size_t)tok * M + m] = gate[tok] * v;
    }
  }
  }
}

}  // namespace

cudaError_t launch_expert_gemm_f32(const Shape& s, const Workspace& ws, int which, const void* W,
                                   const void* bias, const float* gate, void* out,
                                   cudaStream_t stream) {
  const int M = static_cast<int>(which == 0 ? s.d_ff : s.d);
  const int K = static_cast<int>(which == 0 ? s.d : s.d_ff);
  const float* act = static_cast<const float*>(which == 0 ? ws.xbuf : ws.hbuf);
  // upper bound on row tiles: sum_e ceil(m_e / 32) <= A / 32 + N (A = T * topk rows)
  const int64_t max_tiles = (packed_rows(s) + kTile - 1) / kTile + s.N;
  dim3 grid(static_cast<unsigned>(max_tiles), (M + kTile - 1) / kTile);
  const bool glu = which == 0 && s.glu;
  const cudaError_t e = launch_dependent(
      glu ? expert_gemm_f32_kernel<true> : expert_gemm_f32_kernel<false>, grid, dim3(256), 0,
      stream, act, static_cast<const float*>(W),
      static_cast<const float*>(bias), static_cast<const int*>(ws.tile_prefix),
      static_cast<const int*>(ws.exp_rows), static_cast<const int*>(ws.exp_base),
      static_cast<const int*>(ws.slot_token), gate, static_cast<float*>(out),
      static_cast<int>(s.N), M, K, which == 1 && gate == nullptr ? 2 : which,
      static_cast<int>(packed_rows(s)), &ws.hdr->err);
  count_launch();
  return e;
}

}  // namespace swl
