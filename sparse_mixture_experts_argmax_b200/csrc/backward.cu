// Backward pass of the Switch layer (top-1, ReLU experts).
//
// The gradient reaches the router only through the gate: the chosen expert's
// output is scaled by its router probability, so dL/dp_e = dout . u with
// u = E_e(x) ("Switch Transformer, explained", "Why one expert is enough").
// The load-balancing loss N sum_i f_i P_i passes its gradient through P_i only;
// f_i is a count (paper-graph summary of arXiv 2101.03961, "The loss
// formulation").  The argmax, the positions and the capacity cut are piecewise
// constant and pass nothing.  For a kept token t of expert e with gate g,
// a = W1[e] x + b1[e], h = relu(a), u = W2[e] h + b2[e]:
//   du = g dout_t                dW2[e] += du h^T        db2[e] += du
//   da = (W2[e]^T du) * [h > 0]  dW1[e] += da x^T        db1[e] += da
//   dx_t += W1[e]^T da           dg_t = dout_t . u = (dout_t . out_t) / g
// and for every token, with p_t = softmax(W_r x_t + b_r) recomputed in fp32:
//   dz_t,j = dg_t g (delta_{j e} - p_t,j) [kept t]
//          + daux (N / T) p_t,j (f_j - sum_i f_i p_t,i)
//   dW_r += dz_t x_t^T, db_r += dz_t, dx_t += W_r^T dz_t.
//
// Kernels:
//   bwd_gate_kernel     per token: dg (fp32), the packed row du = g dout, f counts
//   bwd_logits_kernel   z = x W_r^T + b_r (fp32, [T, N]): tiles of 128 tokens x 64 experts
//   bwd_dz_kernel       per token (a warp): softmax of z, dz in place of z
//   bwd_dwr_kernel      dW_r partials over row chunks (64 experts x 128 columns tiles)
//   bwd_dx_router_kernel dx = (experts' part) + dz W_r, rounded once to the activation type
//   grouped_gemm_kernel SIMT tiles with fp32 accumulation over packed row
//                       groups (one group per expert), two forms:
//                       WGRAD  C[g] = sum over the group's rows of A_r^T B_r
//                       DGRAD  C_r  = A_r W[g] (+ an epilogue per use)
//   colsum_*_kernel     db[g] = sum over the group's rows of A_r (split, then summed)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "kernels.h"

namespace swl {
namespace {

template <typename T>
__device__ __forceinline__ float ld(const T* p) { return static_cast<float>(*p); }
template <typename T>
__device__ __forceinline__ T cvt(float v) { return static_cast<T>(v); }

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = kBwdThreads / 32;

// dg_t = (dout_t . out_t) / g_t for kept tokens (0 for dropped ones), the
// packed row du[r] = g_t dout_t (r = the token's packed row), and the argmax
// counts of f.  One warp per token.
template <typename TA>
__global__ void __launch_bounds__(kBwdThreads)
bwd_gate_kernel(const TA* __restrict__ dout, const TA* __restrict__ out,
                const int* __restrict__ expert_idx, const float* __restrict__ gate,
                const int* __restrict__ pos_in_expert, const int* __restrict__ exp_base,
                int T, int d, int C_cmp, float* __restrict__ dg, TA* __restrict__ du,
                int* __restrict__ counts) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kBwdWarps + warp;
  if (t >= T) return;
  const int e = expert_idx[t];
  if (lane == 0) atomicAdd(&counts[e], 1);
  const int pos = pos_in_expert[t];
  if (pos >= C_cmp) {
    if (lane == 0) dg[t] = 0.f;
    return;
  }
  const float g = gate[t];
  const TA* dy = dout + static_cast<size_t>(t) * d;
  const TA* y = out + static_cast<size_t>(t) * d;
  TA* u = du + static_cast<size_t>(exp_base[e] + pos) * d;
  float acc = 0.f;
  for (int j = lane; j < d; j += 32) {
    const float a = ld(dy + j);
    acc += a * ld(y + j);
    u[j] = cvt<TA>(g * a);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) dg[t] = acc / g;
}

// Tiled SIMT GEMM over groups of packed rows, fp32 accumulation.  64 x 64
// outputs per CTA, 256 threads with 4 x 4 each, K staged through shared memory
// in steps of 16.
//   WGRAD (kWgrad = true): group g owns rows [base[g], base[g] + rows[g]) of A
//     [*, P] and B [*, Q]; C[g] [P, Q] = sum over those rows r of A[r]^T B[r]
//     (C written, not accumulated).  Grid: (Q/64, P/64, groups).  With base =
//     nullptr and groups > 1, group g is the chunk [g K, (g + 1) K) of rows0
//     rows (partial products of one long sum, added by colsum_finish_kernel).
//   DGRAD: C[r] [Q] = A[r] [K] x W[g] [K, Q] for the group's rows; the epilogue
//     by `epi`: 0 store; 1 multiply by [mask[r] > 0] and store (da from dh);
//     2 add into the fp32 accumulator row dst_row[r] (dx).  Grid: (Q/64,
//     row tiles of 64 listed by tile_prefix, 1).
// A single group with base = nullptr covers rows [0, rows0).
constexpr int kGT = 64, kGK = 16;

template <typename TAin, typename TBin, typename TC, bool kWgrad>
__global__ void __launch_bounds__(256)
grouped_gemm_kernel(const TAin* __restrict__ A, const TBin* __restrict__ B, TC* __restrict__ C,
                    int P, int Q, int K, const int* __restrict__ base,
                    const int* __restrict__ rows, int rows0, const int* __restrict__ tile_prefix,
                    int groups, int epi, const TC* __restrict__ mask,
                    const int* __restrict__ dst_row, float* __restrict__ acc_out) {
  __shared__ float As[kGK][kGT + 1];
  __shared__ float Bs[kGK][kGT + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  int g, r0, nr;
  int m0, n0 = blockIdx.x * kGT;
  if (kWgrad) {
    g = blockIdx.z;
    if (base == nullptr && groups > 1) {   // one group of rows0 rows cut into chunks of K
      r0 = g * K;
      nr = max(0, min(K, rows0 - r0));
    } else {
      r0 = base ? base[g] : 0;
      nr = rows ? rows[g] : rows0;
    }
    m0 = blockIdx.y * kGT;
    if (nr == 0) {      // an expert with no kept rows has a zero gradient
      for (int i = threadIdx.x; i < kGT * kGT; i += 256) {
        const int mm = m0 + i / kGT, nn = n0 + i % kGT;
        if (mm < P && nn < Q) C[(static_cast<size_t>(g) * P + mm) * Q + nn] = cvt<TC>(0.f);
      }
      return;
    }
    // C[m][n] = sum_r A[r0 + r][m] B[r0 + r][n]
    for (int k0 = 0; k0 < nr; k0 += kGK) {
      for (int i = threadIdx.x; i < kGK * kGT; i += 256) {
        const int kk = i / kGT, mm = i % kGT;
        const int r = k0 + kk;
        As[kk][mm] = (r < nr && m0 + mm < P) ? ld(A + static_cast<size_t>(r0 + r) * P + m0 + mm)
                                             : 0.f;
        Bs[kk][mm] = (r < nr && n0 + mm < Q) ? ld(B + static_cast<size_t>(r0 + r) * Q + n0 + mm)
                                             : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kGK; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[i] = As[kk][ty * 4 + i];
          b[i] = Bs[kk][tx * 4 + i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int mm = m0 + ty * 4 + i;
      if (mm >= P) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int nn = n0 + tx * 4 + j;
        if (nn < Q) C[(static_cast<size_t>(g) * P + mm) * Q + nn] = cvt<TC>(acc[i][j]);
      }
    }
    return;
  }
  // DGRAD: row tile blockIdx.y of the tile list
  const int tile = blockIdx.y;
  if (tile_prefix) {
    if (tile >= tile_prefix[groups]) return;
    int lo = 0, hi = groups;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tile_prefix[mid] <= tile) lo = mid; else hi = mid;
    }
    g = lo;
    const int nt = tile - tile_prefix[g];
    r0 = base[g] + nt * kGT;
    nr = min(kGT, rows[g] - nt * kGT);
  } else {
    g = 0;
    r0 = tile * kGT;
    nr = min(kGT, rows0 - r0);
    if (nr <= 0) return;
  }
  const TBin* W = B + static_cast<size_t>(g) * K * Q;
  for (int k0 = 0; k0 < K; k0 += kGK) {
    for (int i = threadIdx.x; i < kGK * kGT; i += 256) {
      const int kk = i % kGK, rr = i / kGK;            // A: rows along i / kGK
      As[kk][rr] = (rr < nr && k0 + kk < K) ? ld(A + static_cast<size_t>(r0 + rr) * K + k0 + kk)
                                            : 0.f;
      const int kb = i / kGT, nn = i % kGT;
      Bs[kb][nn] = (k0 + kb < K && n0 + nn < Q) ? ld(W + static_cast<size_t>(k0 + kb) * Q + n0 + nn)
                                                : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = ty * 4 + i;
    if (rr >= nr) continue;
    const int r = r0 + rr;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int nn = n0 + tx * 4 + j;
      if (nn >= Q) continue;
      const size_t o = static_cast<size_t>(r) * Q + nn;
      if (epi == 0) {
        C[o] = cvt<TC>(acc[i][j]);
      } else if (epi == 1) {
        C[o] = cvt<TC>(ld(mask + o) > 0.f ? acc[i][j] : 0.f);
      } else {
        const int t = dst_row ? dst_row[r] : r;
        acc_out[static_cast<size_t>(t) * Q + nn] += acc[i][j];
      }
    }
  }
}

// Router logits for the backward, z = x W_r^T + b_r in fp32 ([T, N], written to
// dz and turned into dz by bwd_dz_kernel): 128 tokens x 64 experts per CTA,
// 256 threads with 8 tokens x 4 experts each, K in steps of 16 through shared
// memory (both tiles k-major, read as 16-byte vectors), so W_r is read once per
// token tile.  vec: d % 4 == 0 with 16-byte aligned W_r and 4-element aligned x
// rows, then each thread loads 4 consecutive k of a token row and of an expert
// row at once; else element by element.
constexpr int kLT = 128, kLN = 64, kLK = 16;

// A thread's 4 consecutive elements of a row at src (zeros when !ok), as fp32.
template <typename T>
__device__ __forceinline__ float4 ld4(const T* src, bool ok) {
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!ok) return r;
  if constexpr (std::is_same<T, float>::value) {
    r = *reinterpret_cast<const float4*>(src);
  } else {
    const uint2 v = *reinterpret_cast<const uint2*>(src);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
    r = make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
  }
  return r;
}

// The three router-gradient products below share one scheme: a 128 x 64 (or 64
// x 128) output tile per CTA, 8 x 4 (or 4 x 8) outputs per thread, K in steps
// of 16.  With vec (every row 4-element aligned), two shared-memory buffers: a
// thread's loads of step k+1 are issued into registers before step k is
// computed and stored to the other buffer after it, so one barrier per step
// separates the steps and the loads overlap the FMAs; otherwise one buffer with
// element-wise loads.

// Router logits for the backward, z = x W_r^T + b_r in fp32 ([T, N], written to
// dz and turned into dz by bwd_dz_kernel): 128 tokens x 64 experts per CTA,
// 256 threads with 8 tokens x 4 experts each (both tiles k-major in shared
// memory, read as 16-byte vectors), so W_r is read once per token tile.  vec:
// d % 4 == 0 with 16-byte aligned W_r and 4-element aligned x rows.
template <typename TA>
__global__ void __launch_bounds__(256, 2)
bwd_logits_kernel(const TA* __restrict__ x, const float* __restrict__ W_r,
                  const float* __restrict__ b_r, int T, int d, int N, int vec,
                  float* __restrict__ z) {
  __shared__ __align__(16) float As[2][kLK][kLT + 4];   // [buffer][k][token]
  __shared__ __align__(16) float Bs[2][kLK][kLN + 4];   // [buffer][k][expert]
  const int tid = threadIdx.x;
  const int tn = tid % 16, tt = tid / 16;           // experts 4 tn.., tokens 8 tt..
  const int n0 = blockIdx.x * kLN, t0 = blockIdx.y * kLT;
  float acc[8][4] = {};
  auto compute = [&](int b) {
#pragma unroll
    for (int kk = 0; kk < kLK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[b][kk][tt * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[b][kk][tt * 8 + 4]);
      const float4 w = *reinterpret_cast<const float4*>(&Bs[b][kk][tn * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bb[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
  };
  if (vec) {
    // this thread: x rows r = q / 4 (q = tid, tid + 256), W_r row tid / 4, at k quad kq
    const int kq = (tid % 4) * 4, rx0 = tid / 4, rx1 = rx0 + 64, rw = tid / 4;
    float4 xa0, xa1, wb;
    auto fetch = [&](int k0) {
      const bool kok = k0 + kq < d;
      xa0 = ld4(x + static_cast<size_t>(t0 + rx0) * d + k0 + kq, kok && t0 + rx0 < T);
      xa1 = ld4(x + static_cast<size_t>(t0 + rx1) * d + k0 + kq, kok && t0 + rx1 < T);
      wb = ld4(W_r + static_cast<size_t>(n0 + rw) * d + k0 + kq, kok && n0 + rw < N);
    };
    auto stash = [&](int b) {
      As[b][kq][rx0] = xa0.x; As[b][kq + 1][rx0] = xa0.y;
      As[b][kq + 2][rx0] = xa0.z; As[b][kq + 3][rx0] = xa0.w;
      As[b][kq][rx1] = xa1.x; As[b][kq + 1][rx1] = xa1.y;
      As[b][kq + 2][rx1] = xa1.z; As[b][kq + 3][rx1] = xa1.w;
      Bs[b][kq][rw] = wb.x; Bs[b][kq + 1][rw] = wb.y;
      Bs[b][kq + 2][rw] = wb.z; Bs[b][kq + 3][rw] = wb.w;
    };
    fetch(0);
    stash(0);
    __syncthreads();
    int b = 0;
    for (int k0 = 0; k0 < d; k0 += kLK, b ^= 1) {
      const bool more = k0 + kLK < d;
      if (more) fetch(k0 + kLK);
      compute(b);
      if (more) stash(b ^ 1);
      __syncthreads();
    }
  } else {
    for (int k0 = 0; k0 < d; k0 += kLK) {
      for (int i = tid; i < kLK * kLT; i += 256) {
        const int kk = i % kLK, r = i / kLK;
        As[0][kk][r] = (t0 + r < T && k0 + kk < d) ? ld(x + static_cast<size_t>(t0 + r) * d + k0 + kk)
                                                   : 0.f;
      }
      for (int i = tid; i < kLK * kLN; i += 256) {
        const int kk = i % kLK, r = i / kLK;
        Bs[0][kk][r] = (n0 + r < N && k0 + kk < d) ? W_r[static_cast<size_t>(n0 + r) * d + k0 + kk]
                                                   : 0.f;
      }
      __syncthreads();
      compute(0);
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + tt * 8 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tn * 4 + j;
      if (n < N) z[static_cast<size_t>(t) * N + n] = acc[i][j] + (b_r ? b_r[n] : 0.f);
    }
  }
}

// dW_r partial products over row chunks: part[s][n][c] = sum over the rows r of
// chunk s (rows [s K, s K + K) of T) of dz[r][n] x[r][c], fp32; 64 experts x 128
// columns per CTA, 256 threads with 4 experts x 8 columns each, rows in steps of
// 16 through shared memory (both tiles row-major as read).  vec: N % 4 == 0 and
// d % 4 == 0 with 16-byte aligned dz and 4-element aligned x.  The chunks are
// then added in order by colsum_finish_kernel.
constexpr int kRN = 64, kRC = 128;
template <typename TA>
__global__ void __launch_bounds__(256, 2)
bwd_dwr_kernel(const float* __restrict__ dz, const TA* __restrict__ x, int T, int d, int N,
               int K, int vec, float* __restrict__ part) {
  __shared__ __align__(16) float As[2][kLK][kRN + 4];   // [buffer][row][expert]
  __shared__ __align__(16) float Bs[2][kLK][kRC + 4];   // [buffer][row][column]
  const int tid = threadIdx.x;
  const int tn = tid % 16, tc = tid / 16;           // experts 4 tn.., columns 8 tc..
  const int c0 = blockIdx.x * kRC, n0 = blockIdx.y * kRN, sidx = blockIdx.z;
  const int r0 = sidx * K, r1 = min(T, r0 + K);
  float acc[4][8] = {};
  auto compute = [&](int b) {
#pragma unroll
    for (int kk = 0; kk < kLK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&As[b][kk][tn * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[b][kk][tc * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[b][kk][tc * 8 + 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[j][i] = fmaf(av[j], bv[i], acc[j][i]);
    }
  };
  if (vec) {
    // this thread: dz row tid / 16 at expert quad nq; x rows q / 32 (q = tid, tid + 256)
    // at column quad cq
    const int kr = tid / 16, nq = (tid % 16) * 4;
    const int xr0 = tid / 32, xr1 = xr0 + 8, cq = (tid % 32) * 4;
    float4 av, xb0, xb1;
    auto fetch = [&](int k0) {
      av = ld4(dz + static_cast<size_t>(k0 + kr) * N + n0 + nq, k0 + kr < r1 && n0 + nq < N);
      const bool cok = c0 + cq < d;
      xb0 = ld4(x + static_cast<size_t>(k0 + xr0) * d + c0 + cq, cok && k0 + xr0 < r1);
      xb1 = ld4(x + static_cast<size_t>(k0 + xr1) * d + c0 + cq, cok && k0 + xr1 < r1);
    };
    auto stash = [&](int b) {
      *reinterpret_cast<float4*>(&As[b][kr][nq]) = av;
      *reinterpret_cast<float4*>(&Bs[b][xr0][cq]) = xb0;
      *reinterpret_cast<float4*>(&Bs[b][xr1][cq]) = xb1;
    };
    fetch(r0);
    stash(0);
    __syncthreads();
    int b = 0;
    for (int k0 = r0; k0 < r1; k0 += kLK, b ^= 1) {
      const bool more = k0 + kLK < r1;
      if (more) fetch(k0 + kLK);
      compute(b);
      if (more) stash(b ^ 1);
      __syncthreads();
    }
  } else {
    for (int k0 = r0; k0 < r1; k0 += kLK) {
      for (int i = tid; i < kLK * kRN; i += 256) {
        const int kr = i / kRN, n = i % kRN;
        As[0][kr][n] = (k0 + kr < r1 && n0 + n < N) ? dz[static_cast<size_t>(k0 + kr) * N + n0 + n]
                                                    : 0.f;
      }
      for (int i = tid; i < kLK * kRC; i += 256) {
        const int kr = i / kRC, c = i % kRC;
        Bs[0][kr][c] = (k0 + kr < r1 && c0 + c < d) ? ld(x + static_cast<size_t>(k0 + kr) * d + c0 + c)
                                                    : 0.f;
      }
      __syncthreads();
      compute(0);
      __syncthreads();
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int n = n0 + tn * 4 + j;
    if (n >= N) continue;
    float* dst = part + (static_cast<size_t>(sidx) * N + n) * d;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = c0 + tc * 8 + i;
      if (c < d) dst[c] = acc[j][i];
    }
  }
}

// dx = dx_acc + dz W_r, rounded once to the activation type: 128 tokens x 64
// columns per CTA, 256 threads with 8 tokens x 4 columns each, K = N in steps
// of 16 (dz k-major in shared memory, W_r rows as read).  vec: N % 4 == 0 and d %
// 4 == 0 with 16-byte aligned dz, W_r and dx_acc.
template <typename TA>
__global__ void __launch_bounds__(256, 2)
bwd_dx_router_kernel(const float* __restrict__ dz, const float* __restrict__ W_r,
                     const float* __restrict__ dx_acc, int T, int d, int N, int vec,
                     TA* __restrict__ dx) {
  __shared__ __align__(16) float As[2][kLK][kLT + 4];   // [buffer][k][token]
  __shared__ __align__(16) float Bs[2][kLK][kLN + 4];   // [buffer][k][column]
  const int tid = threadIdx.x;
  const int tn = tid % 16, tt = tid / 16;           // columns 4 tn.., tokens 8 tt..
  const int c0 = blockIdx.x * kLN, t0 = blockIdx.y * kLT;
  float acc[8][4] = {};
  auto compute = [&](int b) {
#pragma unroll
    for (int kk = 0; kk < kLK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[b][kk][tt * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[b][kk][tt * 8 + 4]);
      const float4 w = *reinterpret_cast<const float4*>(&Bs[b][kk][tn * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bb[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
  };
  if (vec) {
    // this thread: dz rows q / 4 (q = tid, tid + 256) at k quad kq; W_r row tid / 16
    // at column quad cq
    const int kq = (tid % 4) * 4, rz0 = tid / 4, rz1 = rz0 + 64;
    const int kr = tid / 16, cq = (tid % 16) * 4;
    float4 za0, za1, wb;
    auto fetch = [&](int k0) {
      const bool kok = k0 + kq < N;
      za0 = ld4(dz + static_cast<size_t>(t0 + rz0) * N + k0 + kq, kok && t0 + rz0 < T);
      za1 = ld4(dz + static_cast<size_t>(t0 + rz1) * N + k0 + kq, kok && t0 + rz1 < T);
      wb = ld4(W_r + static_cast<size_t>(k0 + kr) * d + c0 + cq, k0 + kr < N && c0 + cq < d);
    };
    auto stash = [&](int b) {
      As[b][kq][rz0] = za0.x; As[b][kq + 1][rz0] = za0.y;
      As[b][kq + 2][rz0] = za0.z; As[b][kq + 3][rz0] = za0.w;
      As[b][kq][rz1] = za1.x; As[b][kq + 1][rz1] = za1.y;
      As[b][kq + 2][rz1] = za1.z; As[b][kq + 3][rz1] = za1.w;
      *reinterpret_cast<float4*>(&Bs[b][kr][cq]) = wb;
    };
    fetch(0);
    stash(0);
    __syncthreads();
    int b = 0;
    for (int k0 = 0; k0 < N; k0 += kLK, b ^= 1) {
      const bool more = k0 + kLK < N;
      if (more) fetch(k0 + kLK);
      compute(b);
      if (more) stash(b ^ 1);
      __syncthreads();
    }
  } else {
    for (int k0 = 0; k0 < N; k0 += kLK) {
      for (int i = tid; i < kLK * kLT; i += 256) {
        const int kk = i % kLK, r = i / kLK;
        As[0][kk][r] = (t0 + r < T && k0 + kk < N) ? dz[static_cast<size_t>(t0 + r) * N + k0 + kk]
                                                   : 0.f;
      }
      for (int i = tid; i < kLK * kLN; i += 256) {
        const int kr = i / kLN, c = i % kLN;
        Bs[0][kr][c] = (k0 + kr < N && c0 + c < d) ? W_r[static_cast<size_t>(k0 + kr) * d + c0 + c]
                                                   : 0.f;
      }
      __syncthreads();
      compute(0);
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + tt * 8 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tn * 4 + j;
      if (c < d) {
        const size_t o = static_cast<size_t>(t) * d + c;
        dx[o] = cvt<TA>(dx_acc[o] + acc[i][j]);
      }
    }
  }
}

// Router gradient, a warp per token, in place of the logits row z_t:
// p = softmax(z_t), dz_t,j = kg (delta_{j e} - p_j) + daux (N / T) p_j (f_j -
// sum_i f_i p_i) with kg = dg_t g_t (0 for a dropped token), f_j = counts_j / T.
// Three passes over the row: max, then the sums of exp and of f exp, then dz.
__global__ void __launch_bounds__(kBwdThreads)
bwd_dz_kernel(const int* __restrict__ expert_idx, const float* __restrict__ gate,
              const float* __restrict__ dg, const int* __restrict__ counts, int T, int N,
              float daux, float* __restrict__ dz) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kBwdWarps + warp;
  if (t >= T) return;
  float* zt = dz + static_cast<size_t>(t) * N;
  const float invT = 1.0f / static_cast<float>(T);
  float m = -INFINITY;
  for (int n = lane; n < N; n += 32) m = fmaxf(m, zt[n]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float s = 0.f, sf = 0.f;
  for (int n = lane; n < N; n += 32) {
    const float e = expf(zt[n] - m);
    s += e;
    sf += static_cast<float>(counts[n]) * invT * e;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, off);
    sf += __shfl_xor_sync(0xffffffffu, sf, off);
  }
  const float inv = 1.0f / s;
  const float fp = sf * inv;   // sum_i f_i p_i
  const int e = expert_idx[t];
  const float kg = dg[t] * gate[t];
  const float ca = daux * static_cast<float>(N) * invT;
  for (int n = lane; n < N; n += 32) {
    const float p = expf(zt[n] - m) * inv;
    const float f = static_cast<float>(counts[n]) * invT;
    zt[n] = kg * ((n == e ? 1.f : 0.f) - p) + ca * p * (f - fp);
  }
}

// bf16 DGRAD form of grouped_gemm_kernel on the tensor cores: mma.sync
// m16n8k16 with fp32 accumulation, 128 x 128 outputs per CTA, 8 warps of 64 x
// 32, K in steps of 32 staged by cp.async into two shared-memory buffers,
// fragments by ldmatrix.  Same row-tile list, grid (with 128-row tiles) and
// epilogues as the SIMT kernel's DGRAD: A is staged [r][k] (read as is), W[g]
// [k][n] (read transposed).  The bf16 WGRAD form is grouped_wgrad_mma_kernel
// below: there the contraction runs over the group's rows for both operands,
// staged [k][m] and [k][n] and both read transposed.
constexpr int kMT = 128, kMK = 32, kMPad = 8;
constexpr int kMStride = kMT + kMPad;      // [k][128] tiles: row stride in elements
constexpr int kMStrideK = kMK + kMPad;     // [128][k] tile: row stride in elements
constexpr int kDgStages = 4;               // cp.async ring depth of grouped_gemm_mma_kernel
constexpr size_t kDgSmem =
    static_cast<size_t>(kDgStages) * (kMT * kMStrideK + kMK * kMStride) * 2 + 128;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// 16-byte async copy; a false predicate copies nothing and zero-fills
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
               "r"(pred ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(256)
grouped_gemm_mma_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B,
                        __nv_bfloat16* __restrict__ C, int Q, int K,
                        const int* __restrict__ base, const int* __restrict__ rows, int rows0,
                        const int* __restrict__ tile_prefix, int groups, int epi,
                        const __nv_bfloat16* __restrict__ mask, const int* __restrict__ dst_row,
                        float* __restrict__ acc_out) {
  extern __shared__ uint8_t dg_raw[];
  __nv_bfloat16* smem = reinterpret_cast<__nv_bfloat16*>(
      (reinterpret_cast<uintptr_t>(dg_raw) + 127) & ~static_cast<uintptr_t>(127));
  __nv_bfloat16* sA = smem;                                // [kDgStages][kMT][kMStrideK]
  __nv_bfloat16* sB = sA + kDgStages * kMT * kMStrideK;    // [kDgStages][kMK][kMStride]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 2, wn = warp & 3;        // 2 x 4 warps of 64 x 32 outputs
  const int n0 = blockIdx.x * kMT;
  int g, r0, nr;
  {
    const int tile = blockIdx.y;
    if (tile_prefix) {
      if (tile >= tile_prefix[groups]) return;
      int lo = 0, hi = groups;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tile_prefix[mid] <= tile) lo = mid; else hi = mid;
      }
      g = lo;
      const int nt = tile - tile_prefix[g];
      r0 = base[g] + nt * kMT;
      nr = min(kMT, rows[g] - nt * kMT);
    } else {
      g = 0;
      r0 = tile * kMT;
      nr = min(kMT, rows0 - r0);
      if (nr <= 0) return;
    }
  }
  const __nv_bfloat16* W = B + static_cast<size_t>(g) * K * Q;

  // stage one K step of 32 into buffer s (every thread: 2 chunks of A, 2 of B)
  auto load = [&](int s, int k0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = tid + h * 256;
      const int r = c >> 2, kc = (c & 3) * 8;    // A[r0 + r][k0 + kc ...]
      const bool ok = r < nr && k0 + kc < K;
      cp_async16(&sA[(s * kMT + r) * kMStrideK + kc],
                 ok ? A + static_cast<size_t>(r0 + r) * K + k0 + kc : A, ok);
      const int k = c >> 4, nc = (c & 15) * 8;    // W[g][k0 + k][n0 + nc ...]
      const bool okb = k0 + k < K && n0 + nc < Q;
      cp_async16(&sB[(s * kMK + k) * kMStride + nc],
                 okb ? W + static_cast<size_t>(k0 + k) * Q + n0 + nc : B, okb);
    }
  };

  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][j][c] = 0.f;

  // kDgStages-deep ring: K steps kt+1 .. kt+kDgStages-1 are in flight while kt
  // is computed; one commit group per K step (empty past the end), so that
  // waiting until kDgStages-2 groups remain leaves step kt landed
  const int nk = (K + kMK - 1) / kMK;
#pragma unroll
  for (int s = 0; s < kDgStages - 1; ++s) {
    if (s < nk) load(s, s * kMK);
    cp_async_commit();
  }
  for (int kt = 0; kt < nk; ++kt) {
    const int s = kt % kDgStages;
    cp_async_wait<kDgStages - 2>();
    __syncthreads();   // step kt landed for every thread; step kt-1's stage is free
    {
      const int kn = kt + kDgStages - 1;
      if (kn < nk) load(kn % kDgStages, kn * kMK);
      cp_async_commit();
    }
    const __nv_bfloat16* a_s = sA + s * kMT * kMStrideK;
    const __nv_bfloat16* b_s = sB + s * kMK * kMStride;
#pragma unroll
    for (int kk = 0; kk < kMK; kk += 16) {
      uint32_t af[4][4], bf[4][2];
      const int jm = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int mb = wm * 64 + i * 16;   // staged [r][k]
        ldsm_x4(af[i], &a_s[(mb + (lane & 15)) * kMStrideK + kk + (lane >> 4) * 8]);
      }
#pragma unroll
      for (int j2 = 0; j2 < 2; ++j2) {   // two n-fragments of 8 per ldmatrix
        const int nb = wn * 32 + j2 * 16;
        uint32_t t4[4];
        ldsm_x4_t(t4, &b_s[(kk + rr + (jm & 1) * 8) * kMStride + nb + (jm >> 1) * 8]);
        bf[2 * j2][0] = t4[0];
        bf[2 * j2][1] = t4[1];
        bf[2 * j2 + 1][0] = t4[2];
        bf[2 * j2 + 1][1] = t4[3];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_bf16(acc[i][j], af[i], bf[j][0], bf[j][1]);
    }
  }
  cp_async_wait<0>();   // the empty trailing groups, before the CTA exits

  // epilogue: accumulator (i, j, c) -> row wm*64 + i*16 + lane/4 (+8 for c >= 2),
  // column wn*32 + j*8 + (lane%4)*2 (+1 for odd c)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int rl = wm * 64 + i * 16 + (lane >> 2) + hh * 8;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int nn = n0 + wn * 32 + j * 8 + (lane & 3) * 2;
        if (nn >= Q) continue;
        const float v0 = acc[i][j][2 * hh], v1 = acc[i][j][2 * hh + 1];
        if (rl >= nr) continue;
        const int r = r0 + rl;
        const size_t o = static_cast<size_t>(r) * Q + nn;
        if (epi == 0) {
          *reinterpret_cast<__nv_bfloat162*>(C + o) = __floats2bfloat162_rn(v0, v1);
        } else if (epi == 1) {
          const __nv_bfloat162 mk = *reinterpret_cast<const __nv_bfloat162*>(mask + o);
          *reinterpret_cast<__nv_bfloat162*>(C + o) = __floats2bfloat162_rn(
              __bfloat162float(mk.x) > 0.f ? v0 : 0.f, __bfloat162float(mk.y) > 0.f ? v1 : 0.f);
        } else {
          const int t = dst_row ? dst_row[r] : r;
          float* d = acc_out + static_cast<size_t>(t) * Q + nn;
          d[0] += v0;
          d[1] += v1;
        }
      }
    }
  }
}

// Expert weight gradients on the tensor cores, persistent: C[g] = A[rows of
// g]^T B[rows of g] ([P, Q] per expert, bf16 inputs, fp32 accumulation, bf16
// out).  CTA b takes output tiles b, b + gridDim.x, ... of the groups x
// ceil(P/128) x ceil(Q/128) tiles (group-major, then m-tile, then n-tile, so
// the CTAs running together share a group's rows in L2, and a group with many
// rows spreads over every CTA).  A group without rows has a zero gradient: its
// tiles are plain zero stores.  Per tile the same 8 warps of 64 x 32 outputs
// as grouped_gemm_mma_kernel, K (the group's rows) in steps of 32 through two
// cp.async stages; the next tile's first K step is requested before this
// tile's epilogue, which stages the tile in shared memory and writes whole
// 16-byte row pieces.
constexpr int kWgStride = kMT + kMPad;       // epilogue staging row stride (elements)
constexpr size_t kWgSmem =
    (4 * static_cast<size_t>(kMK) * kMStride + static_cast<size_t>(kMT) * kWgStride) * 2 + 128;

__global__ void __launch_bounds__(256)
grouped_wgrad_mma_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B,
                         __nv_bfloat16* __restrict__ C, int P, int Q,
                         const int* __restrict__ base, const int* __restrict__ rows, int groups) {
  extern __shared__ uint8_t wg_raw[];
  __nv_bfloat16* smem = reinterpret_cast<__nv_bfloat16*>(
      (reinterpret_cast<uintptr_t>(wg_raw) + 127) & ~static_cast<uintptr_t>(127));
  __nv_bfloat16* sA = smem;                              // [2][kMK][kMStride]  A rows [k][m]
  __nv_bfloat16* sB = sA + 2 * kMK * kMStride;           // [2][kMK][kMStride]  B rows [k][n]
  __nv_bfloat16* sE = sB + 2 * kMK * kMStride;           // [kMT][kWgStride]    output tile
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 2, wn = warp & 3;
  const int mtP = (P + kMT - 1) / kMT, mtQ = (Q + kMT - 1) / kMT;
  const int total = groups * mtP * mtQ;
  // 16-byte row pieces when every row of C starts 16-byte aligned
  const bool vec = (Q % 8) == 0 && (reinterpret_cast<uintptr_t>(C) & 15) == 0;
  struct Tile { int g, m0, n0, r0, nr; };
  auto decode = [&](int t) {
    Tile c;
    c.g = t / (mtP * mtQ);
    const int rem = t - c.g * mtP * mtQ;
    c.m0 = (rem / mtQ) * kMT;
    c.n0 = (rem % mtQ) * kMT;
    c.r0 = base[c.g];
    c.nr = rows[c.g];
    return c;
  };
  // K step k0 of tile c into stage s (every thread: 2 chunks of A, 2 of B)
  auto load = [&](int s, int k0, const Tile& c) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = tid + h * 256;
      const int k = i >> 4, col = (i & 15) * 8;
      const bool oka = k0 + k < c.nr && c.m0 + col < P;
      cp_async16(&sA[(s * kMK + k) * kMStride + col],
                 oka ? A + static_cast<size_t>(c.r0 + k0 + k) * P + c.m0 + col : A, oka);
      const bool okb = k0 + k < c.nr && c.n0 + col < Q;
      cp_async16(&sB[(s * kMK + k) * kMStride + col],
                 okb ? B + static_cast<size_t>(c.r0 + k0 + k) * Q + c.n0 + col : B, okb);
    }
    cp_async_commit();
  };
  int t = blockIdx.x;
  if (t >= total) return;
  Tile cur = decode(t);
  bool pre = false;          // the current tile's first K step is already requested
  while (true) {
    __nv_bfloat16* Cg = C + static_cast<size_t>(cur.g) * P * Q;
    if (cur.nr == 0) {
      if (vec) {
        for (int i = tid; i < kMT * (kMT / 8); i += 256) {
          const int rr = cur.m0 + i / (kMT / 8), cc = cur.n0 + (i % (kMT / 8)) * 8;
          if (rr < P && cc < Q)
            *reinterpret_cast<uint4*>(Cg + static_cast<size_t>(rr) * Q + cc) =
                make_uint4(0u, 0u, 0u, 0u);
        }
      } else {
        for (int i = tid; i < kMT * kMT; i += 256) {
          const int rr = cur.m0 + i / kMT, cc = cur.n0 + i % kMT;
          if (rr < P && cc < Q) Cg[static_cast<size_t>(rr) * Q + cc] = __float2bfloat16(0.f);
        }
      }
      t += gridDim.x;
      if (t >= total) break;
      cur = decode(t);
      pre = false;
      continue;
    }
    if (!pre) load(0, 0, cur);
    float acc[4][4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][j][c] = 0.f;
    const int nk = (cur.nr + kMK - 1) / kMK;
    for (int kt = 0; kt < nk; ++kt) {
      const int s = kt & 1;
      if (kt + 1 < nk) {
        load(s ^ 1, (kt + 1) * kMK, cur);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const __nv_bfloat16* a_s = sA + s * kMK * kMStride;
      const __nv_bfloat16* b_s = sB + s * kMK * kMStride;
#pragma unroll
      for (int kk = 0; kk < kMK; kk += 16) {
        uint32_t af[4][4], bf[4][2];
        const int jm = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int i = 0; i < 4; ++i) {   // staged [k][m]: (m, k) blocks read transposed
          const int mb = wm * 64 + i * 16;
          ldsm_x4_t(af[i], &a_s[(kk + rr + (jm >> 1) * 8) * kMStride + mb + (jm & 1) * 8]);
        }
#pragma unroll
        for (int j2 = 0; j2 < 2; ++j2) {
          const int nb = wn * 32 + j2 * 16;
          uint32_t t4[4];
          ldsm_x4_t(t4, &b_s[(kk + rr + (jm & 1) * 8) * kMStride + nb + (jm >> 1) * 8]);
          bf[2 * j2][0] = t4[0];
          bf[2 * j2][1] = t4[1];
          bf[2 * j2 + 1][0] = t4[2];
          bf[2 * j2 + 1][1] = t4[3];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) mma_bf16(acc[i][j], af[i], bf[j][0], bf[j][1]);
      }
      __syncthreads();
    }
    // every warp is past its last shared-memory read of the stages: the next
    // tile's first K step goes into stage 0 under this tile's epilogue
    const int tn = t + static_cast<int>(gridDim.x);
    Tile nxt = cur;
    pre = false;
    if (tn < total) {
      nxt = decode(tn);
      if (nxt.nr > 0) {
        load(0, 0, nxt);
        pre = true;
      }
    }
    // accumulator (i, j, c) -> row wm*64 + i*16 + lane/4 (+8 for c >= 2), column
    // wn*32 + j*8 + (lane%4)*2 (+1 for odd c), staged as bf16
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int rl = wm * 64 + i * 16 + (lane >> 2) + hh * 8;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int cl = wn * 32 + j * 8 + (lane & 3) * 2;
          *reinterpret_cast<__nv_bfloat162*>(&sE[rl * kWgStride + cl]) =
              __floats2bfloat162_rn(acc[i][j][2 * hh], acc[i][j][2 * hh + 1]);
        }
      }
    __syncthreads();
    if (vec) {
      for (int i = tid; i < kMT * (kMT / 8); i += 256) {
        const int rl = i / (kMT / 8), cl = (i % (kMT / 8)) * 8;
        const int rr = cur.m0 + rl, cc = cur.n0 + cl;
        if (rr < P && cc < Q)
          *reinterpret_cast<uint4*>(Cg + static_cast<size_t>(rr) * Q + cc) =
              *reinterpret_cast<const uint4*>(&sE[rl * kWgStride + cl]);
      }
    } else {
      for (int i = tid; i < kMT * kMT; i += 256) {
        const int rl = i / kMT, cl = i % kMT;
        const int rr = cur.m0 + rl, cc = cur.n0 + cl;
        if (rr < P && cc < Q) Cg[static_cast<size_t>(rr) * Q + cc] = sE[rl * kWgStride + cl];
      }
    }
    __syncthreads();   // sE is free for the next tile
    if (tn >= total) break;
    t = tn;
    cur = nxt;
  }
}

// Column sums per group, in two passes so that long groups spread over many
// CTAs: partial[s][g][m] = sum of A[r][m] over rows s*R .. s*R + R - 1 of group
// g (R = kColRows), one CTA per 32 columns, group and split, its 8 warps taking
// every 8th row and their sums added in warp order; then colsum_finish_kernel
// adds the splits in order (deterministic).
constexpr int kColRows = 256;
// Rows per partial product of the router's dW_r = dz^T x: enough chunks for ~2048
// CTAs of 64 x 64 outputs, chunks of at least kColRows rows (a multiple of 16).
inline int router_chunk_rows(int64_t T, int64_t N, int64_t d) {
  const int64_t tiles = ((d + 63) / 64) * ((N + 63) / 64);
  int64_t S = (2048 + tiles - 1) / tiles;
  const int64_t smax = (T + kColRows - 1) / kColRows;
  if (S > smax) S = smax;
  if (S < 1) S = 1;
  const int64_t chunk = (T + S - 1) / S;
  return static_cast<int>(chunk < 16 ? 16 : (chunk + 15) / 16 * 16);
}

template <typename TA>
__global__ void __launch_bounds__(256)
colsum_partial_kernel(const TA* __restrict__ A, int P, const int* __restrict__ base,
                      const int* __restrict__ rows, int rows0, int groups,
                      float* __restrict__ partial) {
  __shared__ float red[8][33];
  const int g = blockIdx.y, sp = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int m = blockIdx.x * 32 + lane;
  const int r0 = base ? base[g] : 0, nr = rows ? rows[g] : rows0;
  const int lo = sp * kColRows, hi = min(nr, lo + kColRows);
  float sum = 0.f;
  if (m < P)
    for (int r = lo + warp; r < hi; r += 8) sum += ld(A + static_cast<size_t>(r0 + r) * P + m);
  red[warp][lane] = sum;
  __syncthreads();
  if (warp == 0 && m < P) {
    float t = red[0][lane];
#pragma unroll
    for (int w = 1; w < 8; ++w) t += red[w][lane];
    partial[(static_cast<size_t>(sp) * groups + g) * P + m] = t;
  }
}

// out[i] = sum over s < S of partial[s][i], in order; n = groups * P (or the
// [P, Q] products of a chunked WGRAD).
template <typename TC>
__global__ void __launch_bounds__(256)
colsum_finish_kernel(const float* __restrict__ partial, int S, size_t n, TC* __restrict__ out) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float t = 0.f;
    for (int sp = 0; sp < S; ++sp) t += partial[static_cast<size_t>(sp) * n + i];
    out[i] = cvt<TC>(t);
  }
}

// Row tiles of `tile` packed rows per expert for the DGRAD grid.
__global__ void bwd_tile_prefix_kernel(const int* __restrict__ rows, int N, int tile,
                                       int* __restrict__ prefix) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < N; ++e) {
      prefix[e] = acc;
      acc += (rows[e] + tile - 1) / tile;
    }
    prefix[N] = acc;
  }
}

template <typename TA>
cudaError_t run_backward_t(const Shape& s, const Workspace& fw, const BwdWorkspace& bw,
                           const BwdArgs& a, cudaStream_t stream) {
  const int T = static_cast<int>(s.T), d = static_cast<int>(s.d), d_ff = static_cast<int>(s.d_ff);
  const int N = static_cast<int>(s.N);
  const TA* x = static_cast<const TA*>(a.x);
  cudaError_t e;
  int launches = 0;
  if ((e = cudaMemsetAsync(bw.counts, 0, static_cast<size_t>(N) * 4, stream)) != cudaSuccess)
    return e;
  if ((e = cudaMemsetAsync(bw.dx_acc, 0, static_cast<size_t>(T) * d * 4, stream)) != cudaSuccess)
    return e;
  // dg, du rows, argmax counts
  bwd_gate_kernel<TA><<<(T + kBwdWarps - 1) / kBwdWarps, kBwdThreads, 0, stream>>>(
      static_cast<const TA*>(a.dout), static_cast<const TA*>(a.out), a.expert_idx, a.gate,
      a.pos_in_expert, fw.exp_base, T, d, static_cast<int>(s.C_cmp), bw.dg,
      static_cast<TA*>(bw.du), bw.counts);
  ++launches;
  // router: logits z [T, N] into dz, then dz in place
  {
    const int vec = (d % 4 == 0 && (reinterpret_cast<uintptr_t>(a.W_r) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(x) & (4 * sizeof(TA) - 1)) == 0)
                        ? 1
                        : 0;
    bwd_logits_kernel<TA><<<dim3((N + kLN - 1) / kLN, (T + kLT - 1) / kLT), kBwdThreads, 0,
                            stream>>>(x, a.W_r, a.b_r, T, d, N, vec, bw.dz);
    bwd_dz_kernel<<<(T + kBwdWarps - 1) / kBwdWarps, kBwdThreads, 0, stream>>>(
        a.expert_idx, a.gate, bw.dg, bw.counts, T, N, a.daux, bw.dz);
    launches += 2;
  }
  const dim3 blk(256);
  auto tiles = [](int v) { return static_cast<unsigned>((v + kGT - 1) / kGT); };
  // db[g][m] = sum over the group's rows of A[r][m]: split partials, then their sum
  auto colsum = [&](auto* Ain, int P, const int* gbase, const int* grows, int rows0, int groups,
                    int max_rows, auto* out) {
    using TIn = typename std::remove_cv<typename std::remove_pointer<decltype(Ain)>::type>::type;
    using TOut = typename std::remove_pointer<decltype(out)>::type;
    const int S = max(1, (max_rows + kColRows - 1) / kColRows);
    colsum_partial_kernel<TIn><<<dim3((P + 31) / 32, groups, S), blk, 0, stream>>>(
        Ain, P, gbase, grows, rows0, groups, bw.part);
    const size_t n = static_cast<size_t>(groups) * P;
    size_t nb = (n + 255) / 256;
    if (nb > 8 * 148) nb = 8 * 148;
    colsum_finish_kernel<TOut><<<static_cast<unsigned>(nb), blk, 0, stream>>>(bw.part, S, n, out);
    launches += 2;
  };
  const int C_rows = static_cast<int>(s.C_eff);
  if constexpr (std::is_same<TA, __nv_bfloat16>::value) {
    // bf16 layers: the four expert GEMMs on the tensor cores (128 x 128 tiles)
    auto mt = [](int v) { return static_cast<unsigned>((v + kMT - 1) / kMT); };
    const __nv_bfloat16* du = static_cast<const __nv_bfloat16*>(bw.du);
    const __nv_bfloat16* hb = static_cast<const __nv_bfloat16*>(fw.hbuf);
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(fw.xbuf);
    __nv_bfloat16* da = static_cast<__nv_bfloat16*>(bw.da);
    // dW2[e] = du^T h, db2[e] = sum du
    if ((e = cudaFuncSetAttribute(grouped_wgrad_mma_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kWgSmem))) != cudaSuccess)
      return e;
    int sms = 0, dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
    // persistent: two CTAs per SM (registers), or fewer when the tiles are fewer
    auto wg_grid = [&](int P, int Q) {
      const long long tiles = static_cast<long long>(N) * mt(P) * mt(Q);
      return static_cast<unsigned>(tiles < 2LL * sms ? tiles : 2LL * sms);
    };
    grouped_wgrad_mma_kernel<<<wg_grid(d, d_ff), blk, kWgSmem, stream>>>(
        du, hb, static_cast<__nv_bfloat16*>(a.dW2), d, d_ff, fw.exp_base, fw.exp_rows, N);
    colsum(static_cast<const TA*>(bw.du), d, fw.exp_base, fw.exp_rows, 0, N, C_rows,
           static_cast<TA*>(a.db2));
    // da = (du W2[e]) * [h > 0]
    bwd_tile_prefix_kernel<<<1, 32, 0, stream>>>(fw.exp_rows, N, kMT, bw.tile_prefix);
    const unsigned row_tiles = static_cast<unsigned>((T + kMT - 1) / kMT + N);
    if ((e = cudaFuncSetAttribute(grouped_gemm_mma_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kDgSmem))) != cudaSuccess)
      return e;
    grouped_gemm_mma_kernel<<<dim3(mt(d_ff), row_tiles, 1), blk, kDgSmem, stream>>>(
        du, static_cast<const __nv_bfloat16*>(a.W2), da, d_ff, d, fw.exp_base, fw.exp_rows, 0,
        bw.tile_prefix, N, 1, hb, nullptr, nullptr);
    // dW1[e] = da^T x, db1[e] = sum da
    grouped_wgrad_mma_kernel<<<wg_grid(d_ff, d), blk, kWgSmem, stream>>>(
        da, xb, static_cast<__nv_bfloat16*>(a.dW1), d_ff, d, fw.exp_base, fw.exp_rows, N);
    colsum(static_cast<const TA*>(bw.da), d_ff, fw.exp_base, fw.exp_rows, 0, N, C_rows,
           static_cast<TA*>(a.db1));
    // dx (kept tokens) += da W1[e], rows to tokens
    grouped_gemm_mma_kernel<<<dim3(mt(d), row_tiles, 1), blk, kDgSmem, stream>>>(
        da, static_cast<const __nv_bfloat16*>(a.W1), nullptr, d, d_ff, fw.exp_base,
        fw.exp_rows, 0, bw.tile_prefix, N, 2, nullptr, fw.slot_token, bw.dx_acc);
    launches += 5;
  } else {
  grouped_gemm_kernel<TA, TA, TA, true><<<dim3(tiles(d_ff), tiles(d), N), blk, 0, stream>>>(
      static_cast<const TA*>(bw.du), static_cast<const TA*>(fw.hbuf), static_cast<TA*>(a.dW2), d,
      d_ff, 0, fw.exp_base, fw.exp_rows, 0, nullptr, N, 0, nullptr, nullptr, nullptr);
  colsum(static_cast<const TA*>(bw.du), d, fw.exp_base, fw.exp_rows, 0, N, C_rows,
         static_cast<TA*>(a.db2));
  ++launches;
  // da = (du W2[e]) * [h > 0]   (W2[e] is [d, d_ff]: K = d, Q = d_ff)
  bwd_tile_prefix_kernel<<<1, 32, 0, stream>>>(fw.exp_rows, N, kGT, bw.tile_prefix);
  const unsigned max_row_tiles = static_cast<unsigned>((T + kGT - 1) / kGT + N);
  grouped_gemm_kernel<TA, TA, TA, false><<<dim3(tiles(d_ff), max_row_tiles, 1), blk, 0, stream>>>(
      static_cast<const TA*>(bw.du), static_cast<const TA*>(a.W2), static_cast<TA*>(bw.da), 0,
      d_ff, d, fw.exp_base, fw.exp_rows, 0, bw.tile_prefix, N, 1,
      static_cast<const TA*>(fw.hbuf), nullptr, nullptr);
  launches += 2;
  // dW1[e] = da^T x (packed x rows), db1[e] = sum da
  grouped_gemm_kernel<TA, TA, TA, true><<<dim3(tiles(d), tiles(d_ff), N), blk, 0, stream>>>(
      static_cast<const TA*>(bw.da), static_cast<const TA*>(fw.xbuf), static_cast<TA*>(a.dW1),
      d_ff, d, 0, fw.exp_base, fw.exp_rows, 0, nullptr, N, 0, nullptr, nullptr, nullptr);
  colsum(static_cast<const TA*>(bw.da), d_ff, fw.exp_base, fw.exp_rows, 0, N, C_rows,
         static_cast<TA*>(a.db1));
  ++launches;
  // dx (kept tokens) += da W1[e]   (W1[e] is [d_ff, d]: K = d_ff, Q = d), rows to tokens
  grouped_gemm_kernel<TA, TA, TA, false><<<dim3(tiles(d), max_row_tiles, 1), blk, 0, stream>>>(
      static_cast<const TA*>(bw.da), static_cast<const TA*>(a.W1), static_cast<TA*>(nullptr), 0, d,
      d_ff, fw.exp_base, fw.exp_rows, 0, bw.tile_prefix, N, 2, nullptr, fw.slot_token, bw.dx_acc);
  ++launches;
  }
  // router: dW_r = dz^T x over T rows in chunks (router_chunk_rows; partial
  // products, then their sum in chunk order), db_r = sum dz, dx += dz W_r
  {
    const int chunk = router_chunk_rows(T, N, d);
    const int S = (T + chunk - 1) / chunk;
    const int vec = (N % 4 == 0 && d % 4 == 0 && (reinterpret_cast<uintptr_t>(bw.dz) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(x) & (4 * sizeof(TA) - 1)) == 0)
                        ? 1
                        : 0;
    bwd_dwr_kernel<TA><<<dim3((d + kRC - 1) / kRC, (N + kRN - 1) / kRN, S), blk, 0, stream>>>(
        bw.dz, x, T, d, N, chunk, vec, bw.part);
    const size_t n = static_cast<size_t>(N) * d;
    size_t nb = (n + 255) / 256;
    if (nb > 8 * 148) nb = 8 * 148;
    colsum_finish_kernel<float><<<static_cast<unsigned>(nb), blk, 0, stream>>>(bw.part, S, n,
                                                                              a.dW_r);
    launches += 2;
  }
  if (a.db_r) colsum(static_cast<const float*>(bw.dz), N, nullptr, nullptr, T, 1, T, a.db_r);
  // dx = dx_acc (the experts' part) + dz W_r, rounded once
  {
    const int vec = (N % 4 == 0 && d % 4 == 0 && (reinterpret_cast<uintptr_t>(bw.dz) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(a.W_r) & 15) == 0)
                        ? 1
                        : 0;
    bwd_dx_router_kernel<TA><<<dim3((d + kLN - 1) / kLN, (T + kLT - 1) / kLT), blk, 0, stream>>>(
        bw.dz, a.W_r, bw.dx_acc, T, d, N, vec, static_cast<TA*>(a.dx));
    ++launches;
  }
  count_launch(launches);
  return cudaGetLastError();
}

}  // namespace

size_t backward_workspace_layout(const Shape& s, uintptr_t base, BwdWorkspace* w) {
  const size_t elem = s.dtype == 1 ? 2 : 4;
  const size_t T = static_cast<size_t>(s.T), N = static_cast<size_t>(s.N);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) / 256 * 256;
    return base + o;
  };
  BwdWorkspace b{};
  b.dg = reinterpret_cast<float*>(take(T * 4));
  b.counts = reinterpret_cast<int*>(take(N * 4));
  b.tile_prefix = reinterpret_cast<int*>(take((N + 1) * 4));
  b.dz = reinterpret_cast<float*>(take(T * N * 4));
  b.du = reinterpret_cast<void*>(take(T * static_cast<size_t>(s.d) * elem));
  b.da = reinterpret_cast<void*>(take(T * static_cast<size_t>(s.d_ff) * elem));
  b.dx_acc = reinterpret_cast<float*>(take(T * static_cast<size_t>(s.d) * 4));
  // split partials: the column sums (db1, db2, db_r) and the router's dW_r chunks
  const size_t c_eff = static_cast<size_t>(s.C_eff > 0 ? s.C_eff : 1);
  const size_t s_exp = (c_eff + kColRows - 1) / kColRows;
  const size_t s_rt = (T + kColRows - 1) / kColRows;
  const int ch = router_chunk_rows(s.T, s.N, s.d);
  const size_t s_ch = (T + ch - 1) / ch;
  const size_t dmax = static_cast<size_t>(s.d > s.d_ff ? s.d : s.d_ff);
  size_t part = s_exp * N * dmax;
  if (s_rt * N > part) part = s_rt * N;
  if (s_ch * N * static_cast<size_t>(s.d) > part) part = s_ch * N * static_cast<size_t>(s.d);
  b.part = reinterpret_cast<float*>(take(part * 4));
  if (w) *w = b;
  return off;
}

cudaError_t launch_backward(const Shape& s, const Workspace& fw, const BwdWorkspace& bw,
                            const BwdArgs& a, cudaStream_t stream) {
  return s.dtype == 1 ? run_backward_t<__nv_bfloat16>(s, fw, bw, a, stream)
                      : run_backward_t<float>(s, fw, bw, a, stream);
}

}  // namespace swl
