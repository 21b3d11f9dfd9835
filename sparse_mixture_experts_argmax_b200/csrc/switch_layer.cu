// C-ABI host side of the Switch-layer forward: argument validation, exact
// capacity, workspace layout, TMA descriptors and the launch sequence.
//
// Stage order on the caller's stream (no host synchronisation inside):
//   0 router               fp32 logits + softmax/argmax/gate + block ranks.  bf16
//                          layers: the split of W_r into bf16 pieces, then the
//                          tcgen05 router (router_tc.cu; logits only for N > 128);
//                          fp32 layers or SWL_ROUTER_FFMA: FFMA kernels (router.cu)
//   1 router softmax       N > 128 only: max/argmax/gate, ranks (router.cu)
//   2 dispatch scan        offsets, capacity, aux     (dispatch.cu); for N <= 128
//                          and small batches scan and gather are one kernel here
//   3 dispatch gather      pos, packed expert rows    (dispatch.cu)
//   4 expert FFN           GEMM1 + bias + ReLU, GEMM2 + bias + gate + combine
//                          (one tcgen05 launch: expert_gemm_sm100.cu; fp32: two
//                          launches of expert_gemm_f32.cu)
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "switch_layer.h"
#include "kernels.h"

namespace swl {

static std::atomic<uint64_t> g_launches{0};
static std::atomic<int> g_router_mode{SWL_ROUTER_TENSOR};   // switch_layer_set_router_mode
static std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};
static std::atomic<int> g_stall_test{0};
void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }
unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(); }
bool stall_test_enabled() { return g_stall_test.load() != 0; }

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

size_t workspace_layout(const Shape& s, bool host_io, uintptr_t base, Workspace* ws) {
  const size_t elem = s.dtype == SWL_BF16 ? 2 : 4;
  const size_t T = static_cast<size_t>(s.T), N = static_cast<size_t>(s.N);
  const size_t A = static_cast<size_t>(packed_rows(s));   // packed expert rows
  const bool top2 = s.topk == 2;   // the top-2 router's arrays (also No-Token-Left-Behind)
  const size_t nb = static_cast<size_t>(s.nblk);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return base + o;
  };
  Workspace w{};
  w.hdr = reinterpret_cast<WsHeader*>(take(sizeof(WsHeader)));
  w.logits = reinterpret_cast<float*>(
      take(s.router_path != kRouterWide && s.router_path != kRouterTCWide
               ? 0
               : static_cast<size_t>(s.ksplit_eff) * T * N * 4));
  w.blk_count = reinterpret_cast<int*>(take(nb * N * 4));
  w.blk_count1 = reinterpret_cast<int*>(take(top2 ? nb * N * 4 : 0));
  w.exp_count1 = reinterpret_cast<int*>(take(top2 ? N * 4 : 0));
  w.blk_off = reinterpret_cast<int*>(take(nb * N * 4));
  w.blk_psum = reinterpret_cast<float*>(take(nb * N * 4));
  w.exp_count = reinterpret_cast<int*>(take(N * 4));
  w.exp_rows = reinterpret_cast<int*>(take(N * 4));
  w.exp_base = reinterpret_cast<int*>(take(N * 4));
  w.exp_off = reinterpret_cast<int*>(take(N * 4));
  w.tile_prefix = reinterpret_cast<int*>(take((N + 1) * 4));
  w.psum64 = reinterpret_cast<double*>(take(N * 8));
  w.slot_token = reinterpret_cast<int*>(take(A * 4));
  w.ready = reinterpret_cast<int*>(take((A / 16 + N + 1) * 4));
  const bool split = s.ffn_split > 1;
  w.tile_prefix2 = reinterpret_cast<int*>(take(split ? (N + 1) * 4 : 0));
  w.split_base = reinterpret_cast<int*>(take(split ? N * 4 : 0));
  w.part = reinterpret_cast<float*>(
      take(split ? static_cast<size_t>(kSplitMaxGroups) * s.ffn_split * 128 * s.tile_rows * 4 : 0));
  w.split_grp = reinterpret_cast<int*>(take(split ? static_cast<size_t>(kSplitMaxGroups) * 16 : 0));
  w.split_ready = reinterpret_cast<int*>(
      take(split ? static_cast<size_t>(kSplitMaxGroups) * kSplitFactor * 4 : 0));
  w.w3 = reinterpret_cast<void*>(
      take(s.router_path == kRouterTC || s.router_path == kRouterTCWide
               ? 3 * N * static_cast<size_t>(s.d) * 2
               : 0));
  w.xj = reinterpret_cast<float*>(
      take(s.jitter && !s.xsplit ? T * static_cast<size_t>(s.d) * 4 : 0));
  w.x3 = reinterpret_cast<void*>(take(s.xsplit ? 3 * T * static_cast<size_t>(s.d) * 2 : 0));
  w.xbuf = reinterpret_cast<void*>(take(A * static_cast<size_t>(s.d) * elem));
  w.hbuf = reinterpret_cast<void*>(take(A * static_cast<size_t>(s.d_ff) * elem));
  w.ybuf = reinterpret_cast<void*>(take(top2 && !s.ntlb ? A * static_cast<size_t>(s.d) * elem : 0));
  w.ntlb_rank2 = reinterpret_cast<int*>(take(s.ntlb ? T * 4 : 0));
  w.ntlb_gate = reinterpret_cast<float*>(take(s.ntlb ? T * 4 : 0));
  w.ntlb_rec = reinterpret_cast<void*>(take(s.ntlb ? shard_record_bytes(s.N) : 0));
  if (host_io) {
    w.x_dev = reinterpret_cast<void*>(take(T * static_cast<size_t>(s.d) * elem));
    w.out_dev = reinterpret_cast<void*>(take(T * static_cast<size_t>(s.d) * elem));
    w.idx_dev = reinterpret_cast<int*>(take(T * 4));
    w.gate_dev = reinterpret_cast<float*>(take(T * 4));
    w.pos_dev = reinterpret_cast<int*>(take(T * 4));
    w.aux_dev = reinterpret_cast<float*>(take(4));
  }
  w.total_bytes = off;
  if (ws) *ws = w;
  return off;
}

// ---------------------------------------------------------------- TMA descriptors
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode_tiled() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows, inner] (inner contiguous), box [box_rows, 64], 128-byte swizzle.
static bool make_tmap_bf16(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows,
                           uint32_t box_rows) {
  PFN_encodeTiled enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static int num_sms_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

static bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// Fills Shape; returns SWL_OK or the validation error.
static swl_status make_shape(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype, double cf,
                             Shape* s, int topk = 1, int normalize = 1, int glu = 0,
                             int jitter = 0, int ntlb = 0) {
  if (T < 0 || d <= 0 || d_ff <= 0 || N <= 0) return SWL_ERR_INVALID_ARG;
  // No-Token-Left-Behind routes with the top-2 router (first and second choice,
  // unnormalised gates) and keeps at most one slot per token
  if (ntlb && (topk != 2 || normalize || glu || jitter)) return SWL_ERR_INVALID_ARG;
  if (topk != 1 && topk != 2) return SWL_ERR_INVALID_ARG;
  if (topk == 2 && N < 2) return SWL_ERR_INVALID_ARG;                    // two experts needed
  if (topk == 2 && N > kStreamSoftmaxMaxN) return SWL_ERR_UNSUPPORTED;
  if (dtype != SWL_F32 && dtype != SWL_BF16) return SWL_ERR_INVALID_ARG;
  if (!std::isfinite(cf) || !(cf > 0.0)) return SWL_ERR_INVALID_ARG;
  if (dtype == SWL_BF16 && (d % 8 != 0 || d_ff % 8 != 0)) return SWL_ERR_UNSUPPORTED;
  if (N > kMaxExperts) return SWL_ERR_UNSUPPORTED;
  const int64_t lim = INT32_MAX;
  if (T > lim / 2 || d > lim / 2 || d_ff > lim / 2) return SWL_ERR_UNSUPPORTED;
  if (N * (d > d_ff ? d : d_ff) > lim) return SWL_ERR_UNSUPPORTED;   // TMA row coordinates
  s->T = T;
  s->d = d;
  s->d_ff = d_ff;
  s->N = N;
  s->dtype = dtype;
  // top-k capacity ceil(k cf T / N) = the formula's value for k T tokens (one
  // slot per token for No-Token-Left-Behind: the top-1 capacity)
  s->C = switch_layer_capacity(T * (ntlb ? 1 : topk), N, cf);
  s->C_eff = s->C < T ? s->C : T;   // a token has at most one assignment per expert
  s->T_total = T;
  s->C_cmp = s->C_eff;
  s->sharded = 0;
  s->topk = topk;
  s->ntlb = ntlb ? 1 : 0;
  s->normalize = normalize ? 1 : 0;
  s->glu = glu ? 1 : 0;
  s->jitter = jitter ? 1 : 0;
  if (glu && N * 2 * d_ff > INT32_MAX) return SWL_ERR_UNSUPPORTED;   // TMA row coordinates
  // the tensor-core router serves bf16 layers unless the FFMA router was chosen;
  // a jittered router input (x * noise, fp32) takes the tensor-core logits of
  // the wide path at any N, with x * noise split into bf16 pieces
  const bool tensor_router = dtype == SWL_BF16 && g_router_mode.load() == SWL_ROUTER_TENSOR;
  const RouterPlan rp =
      router_plan(T, d, N, tensor_router ? 1 : 0, topk, jitter && tensor_router ? 1 : 0);
  s->router_path = rp.path;
  s->xsplit = jitter && rp.path == kRouterTCWide ? 1 : 0;
  s->kslice = rp.kslice;
  s->ksplit_eff = rp.ksplit;
  s->tpb = rp.tpb;
  s->nblk = static_cast<int>((T + s->tpb - 1) / s->tpb);
  s->tile_rows = dtype == SWL_BF16 ? bf16_tile_rows(s->C_eff) : kF32TileRows;
  // GEMM2 split over K: bf16 top-1 ReLU layers with full 256-row token tiles and
  // a long GEMM2 reduction (d_ff >= 4096), whose dispatch is the scan kernel
  s->ffn_split = 1;
  if (dtype == SWL_BF16 && topk == 1 && !glu && s->tile_rows == 256 && d_ff >= 4096 &&
      !dispatch_fused_ok(*s))
    s->ffn_split = kSplitFactor;
  return SWL_OK;
}

// Shape of one rank's shard of a global batch of T_total tokens: the kernels
// run over the T local tokens, the capacity comes from T_total.
static swl_status make_shard_shape(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                   int64_t T_total, double cf, Shape* s) {
  swl_status st = make_shape(T, d, d_ff, N, dtype, cf, s);
  if (st != SWL_OK) return st;
  if (T_total < T) return SWL_ERR_INVALID_ARG;
  if (T_total > INT32_MAX / 2) return SWL_ERR_UNSUPPORTED;
  s->T_total = T_total;
  s->C = switch_layer_capacity(T_total, N, cf);
  s->C_eff = s->C < T ? s->C : T;
  s->C_cmp = s->C < T_total ? s->C : T_total;
  s->sharded = 1;
  s->ffn_split = 1;
  s->tile_rows = dtype == SWL_BF16 ? bf16_tile_rows(s->C_eff) : kF32TileRows;
  return SWL_OK;
}

// Expert parallelism: the owner-side region of the workspace, after the
// layout of this rank's own tokens (a shard of the global batch).
struct EpLayout {
  EpPlan plan;
  void* xbuf;   // [max_rows, d] received rows, packed by local expert
  void* hbuf;   // [max_rows, d_ff]
  void* ybuf;   // [max_rows, d] expert outputs (bias, no gate)
  size_t total_bytes;
};

static swl_status ep_check(int64_t N, int world, int rank) {
  if (world < 1 || rank < 0 || rank >= world || N % world != 0) return SWL_ERR_INVALID_ARG;
  return SWL_OK;
}

static EpLayout ep_layout(const Shape& s, int world, int rank, uintptr_t base) {
  EpLayout e{};
  const size_t elem = s.dtype == SWL_BF16 ? 2 : 4;
  size_t off = workspace_layout(s, false, 0, nullptr);
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return base + o;
  };
  const int L = static_cast<int>(s.N / world);
  e.plan.N = s.N;
  e.plan.world = world;
  e.plan.rank = rank;
  e.plan.L = L;
  e.plan.C_cmp = s.C_cmp;
  e.plan.max_rows = static_cast<int64_t>(L) * s.C_cmp;
  e.plan.tile_rows = s.dtype == SWL_BF16 ? bf16_tile_rows(s.C_cmp) : kF32TileRows;
  const size_t WL = static_cast<size_t>(world) * L, R = static_cast<size_t>(e.plan.max_rows);
  e.plan.blk_src = reinterpret_cast<int*>(take(WL * 4));
  e.plan.blk_dst = reinterpret_cast<int*>(take(WL * 4));
  e.plan.blk_n = reinterpret_cast<int*>(take(WL * 4));
  e.plan.rows = reinterpret_cast<int*>(take(static_cast<size_t>(L) * 4));
  e.plan.base = reinterpret_cast<int*>(take(static_cast<size_t>(L) * 4));
  e.plan.tile_prefix = reinterpret_cast<int*>(take(static_cast<size_t>(L + 1) * 4));
  e.plan.ready = reinterpret_cast<int*>(take((R / 16 + L + 1) * 4));
  e.plan.hdr = reinterpret_cast<WsHeader*>(base);   // shared with this rank's own stages
  e.xbuf = reinterpret_cast<void*>(take(R * static_cast<size_t>(s.d) * elem));
  e.hbuf = reinterpret_cast<void*>(take(R * static_cast<size_t>(s.d_ff) * elem));
  e.ybuf = reinterpret_cast<void*>(take(R * static_cast<size_t>(s.d) * elem));
  e.total_bytes = off;
  return e;
}

// Stages 0-1: router logits, softmax, argmax, gate, block ranks and statistics.
// rec(k) records stage event k (a no-op without events).
template <typename Rec>
static swl_status run_routing(const Shape& s, const Workspace& ws, const void* x,
                              const float* W_r, const void* W1, int32_t* expert_idx, float* gate,
                              int32_t* pos_in_expert, const float* b_r, cudaStream_t stream,
                              Rec& rec, const float* router_noise = nullptr) {
  if (s.jitter) {
    // the router sees x * noise (fp32, or its three bf16 pieces); the experts keep x
    if (launch_router_jitter(s, ws, x, router_noise, stream) != cudaSuccess) return SWL_ERR_CUDA;
    x = s.xsplit ? ws.x3 : static_cast<const void*>(ws.xj);
  }
  if (s.router_path == kRouterTC || s.router_path == kRouterTCWide) {
    CUtensorMap tx, tw;
    if (!make_tmap_bf16(&tx, x, s.d, (s.xsplit ? 3 : 1) * s.T, 128) ||
        !make_tmap_bf16(&tw, ws.w3, s.d, 3 * s.N,
                        s.router_path == kRouterTCWide ? 128 : router_tc_padded_experts(s.N)))
      return SWL_ERR_CUDA;
    // the FFN's first tiles stream W1 from its start: fetch a slice into L2 while
    // routing and dispatch run, when the router is a single wave of CTAs (with a
    // second wave the prefetch would compete with that wave's loads)
    const size_t w1_bytes = static_cast<size_t>(s.N) * s.d_ff * s.d * 2;
    const int sms = num_sms_current();
    const int64_t router_ctas = s.router_path == kRouterTC ? (s.T + 127) / 128 * s.ksplit_eff : 0;
    const size_t pf = (W1 != nullptr && router_ctas > 0 && router_ctas <= sms)
                          ? (w1_bytes < kL2PrefetchBytes ? w1_bytes : kL2PrefetchBytes)
                          : 0;
    if (launch_router_tc(s, ws, W_r, tx, tw, b_r, expert_idx, gate, pos_in_expert, W1, pf, sms,
                         stream) != cudaSuccess)
      return SWL_ERR_CUDA;
  } else if (launch_router_logits(s, ws, x, W_r, b_r, expert_idx, gate, pos_in_expert,
                                  stream) != cudaSuccess) {
    return SWL_ERR_CUDA;
  }
  if (!rec(1)) return SWL_ERR_CUDA;
  if (softmax_variant(s) != kSoftmaxFused &&
      launch_router_softmax(s, ws, b_r, expert_idx, gate, pos_in_expert, stream) != cudaSuccess)
    return SWL_ERR_CUDA;
  if (!rec(2)) return SWL_ERR_CUDA;
  return SWL_OK;
}

// Stage 4: both expert GEMMs over the packed rows, combine in the epilogue.
static swl_status run_ffn(const Shape& s, const Workspace& ws, const void* W1, const void* b1,
                          const void* W2, const void* b2, const float* gate, void* out,
                          cudaStream_t stream) {
  if (s.dtype == SWL_BF16) {
    const int sms = num_sms_current();
    if (sms <= 0) return SWL_ERR_CUDA;
    CUtensorMap a1, b1m, a2, b2m;
    if (!make_tmap_bf16(&a1, W1, s.d, s.N * s.d_ff * (s.glu ? 2 : 1), 128) ||
        !make_tmap_bf16(&b1m, ws.xbuf, s.d, packed_rows(s), s.tile_rows) ||
        !make_tmap_bf16(&a2, W2, s.d_ff, s.N * s.d, 128) ||
        !make_tmap_bf16(&b2m, ws.hbuf, s.d_ff, packed_rows(s), s.tile_rows))
      return SWL_ERR_CUDA;
    if (launch_expert_ffn_bf16(s, ws, a1, b1m, a2, b2m, b1, b2, gate, out, sms, stream) !=
        cudaSuccess)
      return SWL_ERR_CUDA;
  } else {
    if (launch_expert_gemm_f32(s, ws, 0, W1, b1, gate, ws.hbuf, stream) != cudaSuccess)
      return SWL_ERR_CUDA;
    if (launch_expert_gemm_f32(s, ws, 1, W2, b2, gate, out, stream) != cudaSuccess)
      return SWL_ERR_CUDA;
  }
  return SWL_OK;
}

static swl_status run_forward(const Shape& s, const Workspace& ws, const void* x,
                              const float* W_r, const void* W1, const void* b1, const void* W2,
                              const void* b2, void* out, int32_t* expert_idx, float* gate,
                              int32_t* pos_in_expert, float* aux_loss, const float* b_r,
                              cudaStream_t stream, void* const* ev,
                              const float* router_noise = nullptr) {
  // Under stream capture the records are made external, so that they become
  // event-record nodes of the graph (timable on replay); otherwise plain records.
  bool capturing = false;
  if (ev != nullptr) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return SWL_ERR_CUDA;
    capturing = cs == cudaStreamCaptureStatusActive;
  }
  auto rec = [&](int k) -> bool {
    if (ev == nullptr) return true;
    cudaEvent_t e = static_cast<cudaEvent_t>(ev[k]);
    return (capturing ? cudaEventRecordWithFlags(e, stream, cudaEventRecordExternal)
                      : cudaEventRecord(e, stream)) == cudaSuccess;
  };
  if (!rec(0)) return SWL_ERR_CUDA;
  swl_status st = run_routing(s, ws, x, W_r, W1, expert_idx, gate, pos_in_expert, b_r, stream,
                              rec, router_noise);
  if (st != SWL_OK) return st;
  if (s.ntlb) {
    // No-Token-Left-Behind: both stages' positions (scan stage), the gather of
    // the kept tokens, then the top-1 FFN with each token's keeping probability
    if (launch_ntlb_positions(s, ws, expert_idx, pos_in_expert, aux_loss, stream) !=
        cudaSuccess)
      return SWL_ERR_CUDA;
    if (!rec(3)) return SWL_ERR_CUDA;
    if (launch_ntlb_gather(s, ws, x, expert_idx, gate, pos_in_expert, out, stream) !=
        cudaSuccess)
      return SWL_ERR_CUDA;
    if (!rec(4)) return SWL_ERR_CUDA;
    st = run_ffn(s, ws, W1, b1, W2, b2, ws.ntlb_gate, out, stream);
    if (st != SWL_OK) return st;
    if (!rec(5)) return SWL_ERR_CUDA;
    return SWL_OK;
  }
  if (dispatch_fused_ok(s)) {
    // one launch for scan and gather (timed in the scan stage; the gather stage is empty)
    if (launch_dispatch_fused(s, ws, x, expert_idx, pos_in_expert, out, aux_loss, stream) !=
        cudaSuccess)
      return SWL_ERR_CUDA;
    if (!rec(3)) return SWL_ERR_CUDA;
  } else {
    if (launch_dispatch_scan(s, ws, aux_loss, nullptr, stream) != cudaSuccess)
      return SWL_ERR_CUDA;
    if (!rec(3)) return SWL_ERR_CUDA;
    if (launch_dispatch_gather(s, ws, x, expert_idx, pos_in_expert, out, stream) != cudaSuccess)
      return SWL_ERR_CUDA;
  }
  if (!rec(4)) return SWL_ERR_CUDA;
  // top-2: the GEMM2 epilogue writes each assignment's gated row to ybuf and
  // the combine kernel adds a token's kept rows
  st = run_ffn(s, ws, W1, b1, W2, b2, gate, s.topk == 2 ? ws.ybuf : out, stream);
  if (st != SWL_OK) return st;
  if (s.topk == 2 && launch_combine_top2(s, ws, pos_in_expert, out, stream) != cudaSuccess)
    return SWL_ERR_CUDA;
  if (!rec(5)) return SWL_ERR_CUDA;
  return SWL_OK;
}

static swl_status validate_io(const Shape& s, const void* x, const float* W_r, const void* W1,
                              const void* b1, const void* W2, const void* b2, const void* out,
                              const void* expert_idx, const void* gate, const void* pos,
                              const void* aux, const void* workspace, size_t workspace_bytes,
                              bool host_io) {
  if (!W_r || !W1 || !b1 || !W2 || !b2 || !aux || !workspace) return SWL_ERR_INVALID_ARG;
  // per-token buffers may be NULL only for an empty batch
  if (s.T > 0 && (!x || !out || !expert_idx || !gate || !pos)) return SWL_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return SWL_ERR_UNSUPPORTED;
  const uintptr_t a = s.dtype == SWL_BF16 ? 16 : 4;
  if (!aligned(W1, a) || !aligned(W2, a) ||
      !aligned(W_r, s.router_path == kRouterTC || s.router_path == kRouterTCWide ? 16 : 4) || !aligned(b1, s.dtype ? 2 : 4) ||
      !aligned(b2, s.dtype ? 2 : 4))
    return SWL_ERR_UNSUPPORTED;
  if (!host_io && (!aligned(x, a) || !aligned(out, a))) return SWL_ERR_UNSUPPORTED;
  if (!aligned(expert_idx, 4) || !aligned(gate, 4) || !aligned(pos, 4) || !aligned(aux, 4))
    return SWL_ERR_UNSUPPORTED;
  if (workspace_bytes < workspace_layout(s, host_io, 0, nullptr)) return SWL_ERR_WORKSPACE;
  return SWL_OK;
}

static swl_status forward_impl(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                               const void* x, const float* W_r, const void* W1, const void* b1,
                               const void* W2, const void* b2, double cf, void* out,
                               int32_t* expert_idx, float* gate, int32_t* pos, float* aux,
                               const float* b_r, void* workspace, size_t workspace_bytes,
                               void* stream_v, void* const* ev, int topk = 1,
                               int normalize = 1, int glu = 0,
                               const float* router_noise = nullptr, int ntlb = 0) {
  Shape s;
  swl_status st = make_shape(T, d, d_ff, N, dtype, cf, &s, topk, normalize, glu,
                             router_noise != nullptr ? 1 : 0, ntlb);
  if (st != SWL_OK) return st;
  st = validate_io(s, x, W_r, W1, b1, W2, b2, out, expert_idx, gate, pos, aux, workspace,
                   workspace_bytes, false);
  if (st != SWL_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  if (T == 0) {
    if (cudaMemsetAsync(aux, 0, sizeof(float), stream) != cudaSuccess) return SWL_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream) != cudaSuccess)
      return SWL_ERR_CUDA;
    if (ev)
      for (int k = 0; k <= SWL_NUM_STAGES; ++k)
        if (cudaEventRecord(static_cast<cudaEvent_t>(ev[k]), stream) != cudaSuccess)
          return SWL_ERR_CUDA;
    return SWL_OK;
  }
  Workspace ws;
  workspace_layout(s, false, reinterpret_cast<uintptr_t>(workspace), &ws);
  if (router_noise != nullptr && !aligned(router_noise, 4)) return SWL_ERR_UNSUPPORTED;
  return run_forward(s, ws, x, W_r, W1, b1, W2, b2, out, expert_idx, gate, pos, aux, b_r, stream,
                     ev, router_noise);
}

// ---------------------------------------------------------------- no-alloc scratch
// Fixed device scratch for switch_layer_forward_noalloc.  In host code the
// symbol is only a stand-in: its device address is looked up once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SWL_NOALLOC_MAX_BYTES];

static void* noalloc_scratch_for_current_device() {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* ptrs[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

}  // namespace swl

using namespace swl;

extern "C" {

int64_t switch_layer_capacity(int64_t T, int64_t N, double cf) {
  if (T < 0 || N <= 0 || !std::isfinite(cf) || !(cf > 0.0)) return -1;
  if (T == 0) return 0;
  // cf = mant * 2^e2 exactly, mant < 2^53
  int e = 0;
  const double m = std::frexp(cf, &e);
  const uint64_t mant = static_cast<uint64_t>(std::ldexp(m, 53));
  const int e2 = e - 53;
  unsigned __int128 num = static_cast<unsigned __int128>(mant) * static_cast<uint64_t>(T);
  if (e2 >= 0) {
    if (e2 >= 127 || (num >> (127 - e2)) != 0) return INT64_MAX;
    num <<= e2;
  } else {
    // ceil(num / (N 2^s)) = ceil(ceil(num / 2^s) / N)
    const int sh = -e2;
    if (sh >= 127) {
      num = 1;   // 0 < num < 2^117 <= 2^sh
    } else {
      const unsigned __int128 one = 1;
      num = (num + ((one << sh) - 1)) >> sh;
    }
  }
  const unsigned __int128 n = static_cast<uint64_t>(N);
  const unsigned __int128 q = (num + n - 1) / n;
  if (q > static_cast<unsigned __int128>(INT64_MAX)) return INT64_MAX;
  return static_cast<int64_t>(q);
}

swl_status switch_layer_workspace_size(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                       double cf, int flags, size_t* bytes) {
  if (!bytes) return SWL_ERR_INVALID_ARG;
  if ((flags & ~(SWL_WS_HOST_IO | SWL_WS_TOP2 | SWL_WS_NTLB)) != 0) return SWL_ERR_INVALID_ARG;
  if ((flags & (SWL_WS_TOP2 | SWL_WS_NTLB)) && (flags & SWL_WS_HOST_IO)) return SWL_ERR_INVALID_ARG;
  if ((flags & SWL_WS_TOP2) && (flags & SWL_WS_NTLB)) return SWL_ERR_INVALID_ARG;
  Shape s;
  const bool ntlb = (flags & SWL_WS_NTLB) != 0;
  const swl_status st = make_shape(T, d, d_ff, N, dtype, cf, &s,
                                   (flags & (SWL_WS_TOP2 | SWL_WS_NTLB)) ? 2 : 1, ntlb ? 0 : 1,
                                   0, 0, ntlb ? 1 : 0);
  if (st != SWL_OK) return st;
  *bytes = workspace_layout(s, (flags & SWL_WS_HOST_IO) != 0, 0, nullptr);
  return SWL_OK;
}

swl_status switch_layer_forward(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                const void* x, const float* W_r, const void* W1, const void* b1,
                                const void* W2, const void* b2, double capacity_factor,
                                void* out, int32_t* expert_idx, float* gate,
                                int32_t* pos_in_expert, float* aux_loss, const float* b_r,
                                void* workspace, size_t workspace_bytes, void* stream) {
  return forward_impl(T, d, d_ff, N, dtype, x, W_r, W1, b1, W2, b2, capacity_factor, out,
                      expert_idx, gate, pos_in_expert, aux_loss, b_r, workspace, workspace_bytes,
                      stream, nullptr);
}

static swl_status variant_args(const swl_variant* v, int* topk, int* normalize, int* glu) {
  *topk = 1;
  *normalize = 1;
  *glu = 0;
  if (v == nullptr) return SWL_OK;
  if (v->top_k != 1 && v->top_k != 2) return SWL_ERR_INVALID_ARG;
  if (v->normalize != 0 && v->normalize != 1) return SWL_ERR_INVALID_ARG;
  if (v->activation != SWL_ACT_RELU && v->activation != SWL_ACT_GEGLU) return SWL_ERR_INVALID_ARG;
  *topk = v->top_k;
  *normalize = v->normalize;
  *glu = v->activation == SWL_ACT_GEGLU ? 1 : 0;
  return SWL_OK;
}

swl_status switch_layer_variant_workspace_size(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                               int dtype, double cf, const swl_variant* v,
                                               size_t* bytes) {
  if (!bytes) return SWL_ERR_INVALID_ARG;
  int topk, normalize, glu;
  swl_status st = variant_args(v, &topk, &normalize, &glu);
  if (st != SWL_OK) return st;
  Shape s;
  st = make_shape(T, d, d_ff, N, dtype, cf, &s, topk, normalize, glu,
                  v != nullptr && v->router_noise != nullptr ? 1 : 0);
  if (st != SWL_OK) return st;
  *bytes = workspace_layout(s, false, 0, nullptr);
  return SWL_OK;
}

swl_status switch_layer_forward_variant(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                        int dtype, const void* x, const float* W_r,
                                        const void* W1, const void* b1, const void* W2,
                                        const void* b2, double capacity_factor, void* out,
                                        int32_t* expert_idx, float* gate,
                                        int32_t* pos_in_expert, float* aux_loss,
                                        const float* b_r, const swl_variant* variant,
                                        void* workspace, size_t workspace_bytes,
                                        void* stream) {
  int topk, normalize, glu;
  const swl_status st = variant_args(variant, &topk, &normalize, &glu);
  if (st != SWL_OK) return st;
  return forward_impl(T, d, d_ff, N, dtype, x, W_r, W1, b1, W2, b2, capacity_factor, out,
                      expert_idx, gate, pos_in_expert, aux_loss, b_r, workspace, workspace_bytes,
                      stream, nullptr, topk, normalize, glu,
                      variant != nullptr ? variant->router_noise : nullptr);
}

swl_status switch_layer_forward_ntlb(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                     const void* x, const float* W_r, const void* W1,
                                     const void* b1, const void* W2, const void* b2,
                                     double capacity_factor, void* out, int32_t* expert_idx,
                                     float* gate, int32_t* pos_in_expert, float* aux_loss,
                                     const float* b_r, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  return forward_impl(T, d, d_ff, N, dtype, x, W_r, W1, b1, W2, b2, capacity_factor, out,
                      expert_idx, gate, pos_in_expert, aux_loss, b_r, workspace, workspace_bytes,
                      stream, nullptr, 2, 0, 0, nullptr, 1);
}

swl_status switch_layer_forward_top2(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                     const void* x, const float* W_r, const void* W1,
                                     const void* b1, const void* W2, const void* b2,
                                     double capacity_factor, int normalize, void* out,
                                     int32_t* expert_idx, float* gate, int32_t* pos_in_expert,
                                     float* aux_loss, const float* b_r, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (normalize != 0 && normalize != 1) return SWL_ERR_INVALID_ARG;
  return forward_impl(T, d, d_ff, N, dtype, x, W_r, W1, b1, W2, b2, capacity_factor, out,
                      expert_idx, gate, pos_in_expert, aux_loss, b_r, workspace, workspace_bytes,
                      stream, nullptr, 2, normalize);
}

swl_status switch_layer_forward_timed(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                      const void* x, const float* W_r, const void* W1,
                                      const void* b1, const void* W2, const void* b2,
                                      double capacity_factor, void* out, int32_t* expert_idx,
                                      float* gate, int32_t* pos_in_expert, float* aux_loss,
                                      const float* b_r, void* workspace, size_t workspace_bytes,
                                      void* stream, void* const* stage_events) {
  if (!stage_events) return SWL_ERR_INVALID_ARG;
  for (int k = 0; k <= SWL_NUM_STAGES; ++k)
    if (!stage_events[k]) return SWL_ERR_INVALID_ARG;
  return forward_impl(T, d, d_ff, N, dtype, x, W_r, W1, b1, W2, b2, capacity_factor, out,
                      expert_idx, gate, pos_in_expert, aux_loss, b_r, workspace, workspace_bytes,
                      stream, stage_events);
}

swl_status switch_layer_forward_host_io(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                        const void* x_host, const float* W_r, const void* W1,
                                        const void* b1, const void* W2, const void* b2,
                                        double capacity_factor, void* out_host,
                                        int32_t* expert_idx_host, float* gate_host,
                                        int32_t* pos_host, float* aux_host, const float* b_r,
                                        void* workspace, size_t workspace_bytes, void* stream_v) {
  Shape s;
  swl_status st = make_shape(T, d, d_ff, N, dtype, capacity_factor, &s);
  if (st != SWL_OK) return st;
  st = validate_io(s, x_host, W_r, W1, b1, W2, b2, out_host, expert_idx_host, gate_host, pos_host,
                   aux_host, workspace, workspace_bytes, true);
  if (st != SWL_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  if (T == 0) {
    *aux_host = 0.f;
    return SWL_OK;
  }
  Workspace ws;
  workspace_layout(s, true, reinterpret_cast<uintptr_t>(workspace), &ws);
  const size_t elem = dtype == SWL_BF16 ? 2 : 4;
  const size_t xb = static_cast<size_t>(T) * static_cast<size_t>(d) * elem;
  const size_t tb = static_cast<size_t>(T) * 4;
  if (cudaMemcpyAsync(ws.x_dev, x_host, xb, cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return SWL_ERR_CUDA;
  st = run_forward(s, ws, ws.x_dev, W_r, W1, b1, W2, b2, ws.out_dev, ws.idx_dev, ws.gate_dev,
                   ws.pos_dev, ws.aux_dev, b_r, stream, nullptr);
  if (st != SWL_OK) return st;
  if (cudaMemcpyAsync(out_host, ws.out_dev, xb, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemcpyAsync(expert_idx_host, ws.idx_dev, tb, cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaMemcpyAsync(gate_host, ws.gate_dev, tb, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemcpyAsync(pos_host, ws.pos_dev, tb, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemcpyAsync(aux_host, ws.aux_dev, 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return SWL_ERR_CUDA;
  return SWL_OK;
}

swl_status switch_layer_device_status(const void* workspace, void* stream) {
  if (!workspace) return SWL_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SWL_ERR_CUDA;
  int err = 0;
  if (cudaMemcpy(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SWL_ERR_CUDA;
  return err == kDevOk ? SWL_OK : SWL_ERR_DEVICE;
}

const char* switch_layer_status_string(swl_status status) {
  switch (status) {
    case SWL_OK: return "ok";
    case SWL_ERR_INVALID_ARG: return "invalid argument";
    case SWL_ERR_UNSUPPORTED: return "unsupported shape, dtype or alignment";
    case SWL_ERR_WORKSPACE: return "workspace too small";
    case SWL_ERR_CUDA: return "CUDA runtime error";
    case SWL_ERR_DEVICE: return "device-side failure reported by a kernel";
  }
  return "unknown status";
}

const char* switch_layer_stage_name(int k) {
  static const char* names[SWL_NUM_STAGES] = {"router_logits", "router_softmax",
                                              "dispatch_scan", "dispatch_gather", "expert_ffn"};
  return (k >= 0 && k < SWL_NUM_STAGES) ? names[k] : nullptr;
}

uint64_t switch_layer_launch_count(void) { return g_launches.load(); }

swl_status switch_layer_set_router_mode(int mode) {
  if (mode != SWL_ROUTER_TENSOR && mode != SWL_ROUTER_FFMA) return SWL_ERR_INVALID_ARG;
  swl::g_router_mode.store(mode);
  return SWL_OK;
}

int switch_layer_router_mode(void) { return swl::g_router_mode.load(); }

swl_status switch_layer_set_wait_limit_ns(uint64_t ns) {
  swl::g_wait_limit_ns.store(ns == 0 ? 2000000000ull : ns);
  return SWL_OK;
}

swl_status switch_layer_set_stall_test(int on) {
  if (on != 0 && on != 1) return SWL_ERR_INVALID_ARG;
  swl::g_stall_test.store(on);
  return SWL_OK;
}

swl_status switch_layer_describe_plan(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                      double capacity_factor, int num_sms, char* buf,
                                      size_t len) {
  if (buf == nullptr || len == 0 || num_sms <= 0) return SWL_ERR_INVALID_ARG;
  Shape s;
  const swl_status st = make_shape(T, d, d_ff, N, dtype, capacity_factor, &s);
  if (st != SWL_OK) return st;
  const char* router = "?";
  switch (s.router_path) {
    case kRouterWarpSplit: router = "ffma_warpsplit"; break;
    case kRouterTile: router = "ffma_tile"; break;
    case kRouterWide: router = "ffma_wide"; break;
    case kRouterTC: router = "tc"; break;
    case kRouterTCWide: router = "tc_wide"; break;
    default: break;
  }
  const bool tc = s.router_path == kRouterTC || s.router_path == kRouterTCWide;
  const bool bf16 = s.dtype == SWL_BF16;
  static const char* const softmax_names[4] = {"fused", "stream", "rows", "wide"};
  char tmp[256];
  const int n = std::snprintf(
      tmp, sizeof(tmp),
      "router=%s,ksplit=%d,router_stages=%d,softmax=%s,tokens_per_block=%d,dispatch=%s,"
      "ffn=%s,tile_rows=%d,accumulators=%d,gemm2_split=%d",
      router, s.ksplit_eff, tc ? router_tc_stages(s, num_sms) : 0,
      softmax_names[softmax_variant(s)], s.tpb,
      dispatch_fused_ok(s) ? "fused" : "two_kernel", bf16 ? "sm100" : "f32", s.tile_rows,
      bf16 ? ffn_accumulators(s.tile_rows) : 0, s.ffn_split);
  if (n < 0 || static_cast<size_t>(n) >= len) return SWL_ERR_INVALID_ARG;
  std::memcpy(buf, tmp, static_cast<size_t>(n) + 1);
  return SWL_OK;
}

swl_status switch_layer_forward_noalloc(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                        const void* x, const float* W_r, const void* W1,
                                        const void* b1, const void* W2, const void* b2,
                                        double capacity_factor, void* out, int32_t* expert_idx,
                                        float* gate, int32_t* pos_in_expert, float* aux_loss,
                                        const float* b_r, void* stream) {
  Shape s;
  const swl_status st = make_shape(T, d, d_ff, N, dtype, capacity_factor, &s);
  if (st != SWL_OK) return st;
  if (workspace_layout(s, false, 0, nullptr) > static_cast<size_t>(SWL_NOALLOC_MAX_BYTES))
    return SWL_ERR_WORKSPACE;   // shape too large for the fixed scratch
  void* scratch = noalloc_scratch_for_current_device();
  if (scratch == nullptr) return SWL_ERR_CUDA;
  return forward_impl(T, d, d_ff, N, dtype, x, W_r, W1, b1, W2, b2, capacity_factor, out,
                      expert_idx, gate, pos_in_expert, aux_loss, b_r, scratch,
                      static_cast<size_t>(SWL_NOALLOC_MAX_BYTES), stream, nullptr);
}

size_t switch_layer_shard_record_bytes(int64_t N) {
  return N > 0 && N <= kMaxExperts ? shard_record_bytes(N) : 0;
}

swl_status switch_layer_forward_shard_begin(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                            int dtype, int64_t T_total, const void* x,
                                            const float* W_r, const float* b_r,
                                            double capacity_factor, int32_t* expert_idx,
                                            float* gate, int32_t* pos_in_expert, void* record,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream_v) {
  Shape s;
  swl_status st = make_shard_shape(T, d, d_ff, N, dtype, T_total, capacity_factor, &s);
  if (st != SWL_OK) return st;
  if (!W_r || !record || !workspace) return SWL_ERR_INVALID_ARG;
  if (T > 0 && (!x || !expert_idx || !gate || !pos_in_expert)) return SWL_ERR_INVALID_ARG;
  const bool tc = s.router_path == kRouterTC || s.router_path == kRouterTCWide;
  if (!aligned(workspace, 256) || !aligned(record, 16) || !aligned(W_r, tc ? 16 : 4) ||
      !aligned(x, dtype == SWL_BF16 ? 16 : 4) || !aligned(expert_idx, 4) || !aligned(gate, 4) ||
      !aligned(pos_in_expert, 4))
    return SWL_ERR_UNSUPPORTED;
  if (workspace_bytes < workspace_layout(s, false, 0, nullptr)) return SWL_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  if (T == 0) {   // no tokens here: an all-zero record
    return cudaMemsetAsync(record, 0, shard_record_bytes(N), stream) == cudaSuccess
               ? SWL_OK
               : SWL_ERR_CUDA;
  }
  Workspace ws;
  workspace_layout(s, false, reinterpret_cast<uintptr_t>(workspace), &ws);
  auto no_events = [](int) { return true; };
  st = run_routing(s, ws, x, W_r, nullptr, expert_idx, gate, pos_in_expert, b_r, stream,
                   no_events);
  if (st != SWL_OK) return st;
  return launch_dispatch_scan(s, ws, nullptr, record, stream) == cudaSuccess ? SWL_OK
                                                                             : SWL_ERR_CUDA;
}

swl_status switch_layer_forward_shard_end(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                          int dtype, int64_t T_total, int rank, int world,
                                          const void* gathered, const void* x, const void* W1,
                                          const void* b1, const void* W2, const void* b2,
                                          double capacity_factor, void* out,
                                          int32_t* expert_idx, float* gate,
                                          int32_t* pos_in_expert, float* aux_loss,
                                          void* workspace, size_t workspace_bytes,
                                          void* stream_v) {
  Shape s;
  swl_status st = make_shard_shape(T, d, d_ff, N, dtype, T_total, capacity_factor, &s);
  if (st != SWL_OK) return st;
  if (world < 1 || rank < 0 || rank >= world) return SWL_ERR_INVALID_ARG;
  if (!gathered || !W1 || !b1 || !W2 || !b2 || !aux_loss || !workspace)
    return SWL_ERR_INVALID_ARG;
  if (T > 0 && (!x || !out || !expert_idx || !gate || !pos_in_expert)) return SWL_ERR_INVALID_ARG;
  const uintptr_t a = dtype == SWL_BF16 ? 16 : 4;
  if (!aligned(workspace, 256) || !aligned(gathered, 16) || !aligned(W1, a) ||
      !aligned(W2, a) || !aligned(b1, dtype == SWL_BF16 ? 2 : 4) ||
      !aligned(b2, dtype == SWL_BF16 ? 2 : 4) || !aligned(x, a) || !aligned(out, a) ||
      !aligned(expert_idx, 4) || !aligned(gate, 4) || !aligned(pos_in_expert, 4) ||
      !aligned(aux_loss, 4))
    return SWL_ERR_UNSUPPORTED;
  if (workspace_bytes < workspace_layout(s, false, 0, nullptr)) return SWL_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  if (T_total == 0) {
    if (cudaMemsetAsync(aux_loss, 0, sizeof(float), stream) != cudaSuccess ||
        cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream) != cudaSuccess)
      return SWL_ERR_CUDA;
    return SWL_OK;
  }
  Workspace ws;
  workspace_layout(s, false, reinterpret_cast<uintptr_t>(workspace), &ws);
  if (T == 0 && cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream) != cudaSuccess)
    return SWL_ERR_CUDA;   // no router ran here to reset the header
  if (launch_shard_combine(s, ws, gathered, rank, world, aux_loss, stream) != cudaSuccess)
    return SWL_ERR_CUDA;
  if (T == 0) return SWL_OK;
  if (launch_dispatch_gather(s, ws, x, expert_idx, pos_in_expert, out, stream) != cudaSuccess)
    return SWL_ERR_CUDA;
  return run_ffn(s, ws, W1, b1, W2, b2, gate, out, stream);
}

int64_t switch_layer_ep_max_recv_rows(int64_t N, int world, int64_t T_total,
                                      double capacity_factor) {
  if (N <= 0 || world < 1 || N % world != 0 || T_total < 0) return -1;
  const int64_t C = switch_layer_capacity(T_total, N, capacity_factor);
  if (C < 0) return -1;
  return (N / world) * (C < T_total ? C : T_total);
}

swl_status switch_layer_ep_workspace_size(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                          int dtype, int world, int64_t T_total,
                                          double capacity_factor, size_t* bytes) {
  if (!bytes) return SWL_ERR_INVALID_ARG;
  swl_status st = ep_check(N, world, 0);
  if (st != SWL_OK) return st;
  Shape s;
  st = make_shard_shape(T, d, d_ff, N, dtype, T_total, capacity_factor, &s);
  if (st != SWL_OK) return st;
  *bytes = ep_layout(s, world, 0, 0).total_bytes;
  return SWL_OK;
}

swl_status switch_layer_ep_counts(int64_t N, int world, int rank, int64_t T_total,
                                  double capacity_factor, const void* gathered_host,
                                  int64_t* send_rows, int64_t* recv_rows) {
  swl_status st = ep_check(N, world, rank);
  if (st != SWL_OK) return st;
  if (!gathered_host || !send_rows || !recv_rows || T_total < 0) return SWL_ERR_INVALID_ARG;
  const int64_t C = switch_layer_capacity(T_total, N, capacity_factor);
  if (C < 0) return SWL_ERR_INVALID_ARG;
  const int64_t C_cmp = C < T_total ? C : T_total;
  const size_t R = shard_record_bytes(N);
  const int64_t L = N / world;
  const uint8_t* g0 = static_cast<const uint8_t*>(gathered_host);
  for (int r = 0; r < world; ++r) send_rows[r] = recv_rows[r] = 0;
  for (int64_t e = 0; e < N; ++e) {
    const int owner = static_cast<int>(e / L);
    int64_t before = 0;
    for (int g = 0; g < world; ++g) {
      int32_t c;
      std::memcpy(&c, g0 + static_cast<size_t>(g) * R + static_cast<size_t>(e) * 4, 4);
      int64_t m = C_cmp - before;
      if (m < 0) m = 0;
      if (m > c) m = c;
      if (g == rank) send_rows[owner] += m;       // my kept rows of e go to its owner
      if (owner == rank) recv_rows[g] += m;       // g's kept rows of my expert e
      before += c;
    }
  }
  return SWL_OK;
}

swl_status switch_layer_ep_dispatch(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                    int world, int rank, int64_t T_total,
                                    double capacity_factor, const void* gathered, const void* x,
                                    int32_t* expert_idx, int32_t* pos_in_expert,
                                    float* aux_loss, void* send_rows, void* workspace,
                                    size_t workspace_bytes, void* stream_v) {
  swl_status st = ep_check(N, world, rank);
  if (st != SWL_OK) return st;
  Shape s;
  st = make_shard_shape(T, d, d_ff, N, dtype, T_total, capacity_factor, &s);
  if (st != SWL_OK) return st;
  if (!gathered || !aux_loss || !workspace) return SWL_ERR_INVALID_ARG;
  if (T > 0 && (!x || !expert_idx || !pos_in_expert || !send_rows)) return SWL_ERR_INVALID_ARG;
  const uintptr_t a = dtype == SWL_BF16 ? 16 : 4;
  if (!aligned(workspace, 256) || !aligned(gathered, 16) || !aligned(x, a) ||
      !aligned(send_rows, a) || !aligned(expert_idx, 4) || !aligned(pos_in_expert, 4) ||
      !aligned(aux_loss, 4))
    return SWL_ERR_UNSUPPORTED;
  if (workspace_bytes < ep_layout(s, world, rank, 0).total_bytes) return SWL_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  if (T_total == 0) {
    return cudaMemsetAsync(aux_loss, 0, sizeof(float), stream) == cudaSuccess ? SWL_OK
                                                                              : SWL_ERR_CUDA;
  }
  Workspace ws;
  workspace_layout(s, false, reinterpret_cast<uintptr_t>(workspace), &ws);
  if (T == 0 && cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream) != cudaSuccess)
    return SWL_ERR_CUDA;
  if (launch_shard_combine(s, ws, gathered, rank, world, aux_loss, stream) != cudaSuccess)
    return SWL_ERR_CUDA;
  if (T == 0) return SWL_OK;
  // this rank's kept rows, packed by expert: the send buffer (experts of one
  // owner are consecutive, so each owner's rows form one segment)
  Workspace wsend = ws;
  wsend.xbuf = send_rows;
  return launch_dispatch_gather(s, wsend, x, expert_idx, pos_in_expert, nullptr, stream) ==
                 cudaSuccess
             ? SWL_OK
             : SWL_ERR_CUDA;
}

swl_status switch_layer_ep_experts(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                   int world, int rank, int64_t T_total, double capacity_factor,
                                   const void* gathered, void* recv_rows, int64_t n_recv,
                                   const void* W1_local, const void* b1_local,
                                   const void* W2_local, const void* b2_local, void* ret_rows,
                                   void* workspace, size_t workspace_bytes, void* stream_v) {
  swl_status st = ep_check(N, world, rank);
  if (st != SWL_OK) return st;
  Shape s;
  st = make_shard_shape(T, d, d_ff, N, dtype, T_total, capacity_factor, &s);
  if (st != SWL_OK) return st;
  if (!gathered || !W1_local || !b1_local || !W2_local || !b2_local || !workspace || n_recv < 0)
    return SWL_ERR_INVALID_ARG;
  if (n_recv > 0 && (!recv_rows || !ret_rows)) return SWL_ERR_INVALID_ARG;
  const uintptr_t a = dtype == SWL_BF16 ? 16 : 4;
  if (!aligned(workspace, 256) || !aligned(gathered, 16) || !aligned(recv_rows, a) ||
      !aligned(ret_rows, a) || !aligned(W1_local, a) || !aligned(W2_local, a))
    return SWL_ERR_UNSUPPORTED;
  const EpLayout ep = ep_layout(s, world, rank, reinterpret_cast<uintptr_t>(workspace));
  if (workspace_bytes < ep.total_bytes) return SWL_ERR_WORKSPACE;
  if (n_recv > ep.plan.max_rows) return SWL_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  if (T_total == 0 || ep.plan.max_rows == 0) return SWL_OK;
  const int row_bytes = static_cast<int>(d * (dtype == SWL_BF16 ? 2 : 4));
  if (launch_ep_plan(ep.plan, gathered, stream) != cudaSuccess) return SWL_ERR_CUDA;
  if (launch_ep_permute(ep.plan, recv_rows, ep.xbuf, n_recv, row_bytes, 0, stream) !=
      cudaSuccess)
    return SWL_ERR_CUDA;
  // the owner's experts over their packed rows: an ordinary FFN of L experts
  // and max_rows rows whose GEMM2 writes bias-added packed rows (no gate)
  Shape so = s;
  so.T = ep.plan.max_rows;
  so.N = ep.plan.L;
  so.topk = 1;
  so.ffn_split = 1;
  so.tile_rows = ep.plan.tile_rows;
  Workspace wo{};
  wo.hdr = ep.plan.hdr;
  wo.tile_prefix = ep.plan.tile_prefix;
  wo.exp_rows = ep.plan.rows;
  wo.exp_base = ep.plan.base;
  wo.ready = ep.plan.ready;
  wo.xbuf = ep.xbuf;
  wo.hbuf = ep.hbuf;
  st = run_ffn(so, wo, W1_local, b1_local, W2_local, b2_local, nullptr, ep.ybuf, stream);
  if (st != SWL_OK) return st;
  return launch_ep_permute(ep.plan, ret_rows, ep.ybuf, n_recv, row_bytes, 1, stream) ==
                 cudaSuccess
             ? SWL_OK
             : SWL_ERR_CUDA;
}

swl_status switch_layer_ep_combine(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                   int world, int rank, int64_t T_total,
                                   double capacity_factor, const void* ret_rows,
                                   const int32_t* expert_idx, const float* gate,
                                   const int32_t* pos_in_expert, void* out, void* workspace,
                                   size_t workspace_bytes, void* stream_v) {
  swl_status st = ep_check(N, world, rank);
  if (st != SWL_OK) return st;
  Shape s;
  st = make_shard_shape(T, d, d_ff, N, dtype, T_total, capacity_factor, &s);
  if (st != SWL_OK) return st;
  if (!workspace) return SWL_ERR_INVALID_ARG;
  if (T > 0 && (!ret_rows || !expert_idx || !gate || !pos_in_expert || !out))
    return SWL_ERR_INVALID_ARG;
  const uintptr_t a = dtype == SWL_BF16 ? 16 : 4;
  if (!aligned(workspace, 256) || !aligned(ret_rows, a) || !aligned(out, a))
    return SWL_ERR_UNSUPPORTED;
  if (workspace_bytes < ep_layout(s, world, rank, 0).total_bytes) return SWL_ERR_WORKSPACE;
  Workspace ws;
  workspace_layout(s, false, reinterpret_cast<uintptr_t>(workspace), &ws);
  return launch_ep_combine(s, ws, ret_rows, expert_idx, gate, pos_in_expert, out,
                           static_cast<cudaStream_t>(stream_v)) == cudaSuccess
             ? SWL_OK
             : SWL_ERR_CUDA;
}

swl_status switch_layer_backward_workspace_size(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                                int dtype, double capacity_factor,
                                                size_t* bytes) {
  if (!bytes) return SWL_ERR_INVALID_ARG;
  Shape s;
  const swl_status st = make_shape(T, d, d_ff, N, dtype, capacity_factor, &s);
  if (st != SWL_OK) return st;
  *bytes = backward_workspace_layout(s, 0, nullptr);
  return SWL_OK;
}

swl_status switch_layer_backward(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                 const void* x, const float* W_r, const float* b_r,
                                 const void* W1, const void* b1, const void* W2, const void* b2,
                                 double capacity_factor, const void* out,
                                 const int32_t* expert_idx, const float* gate,
                                 const int32_t* pos_in_expert, const void* fwd_workspace,
                                 size_t fwd_workspace_bytes, const void* dout, float daux,
                                 void* dx, float* dW_r, float* db_r, void* dW1, void* db1,
                                 void* dW2, void* db2, void* bwd_workspace,
                                 size_t bwd_workspace_bytes, void* stream) {
  Shape s;
  swl_status st = make_shape(T, d, d_ff, N, dtype, capacity_factor, &s);
  if (st != SWL_OK) return st;
  if (!W_r || !W1 || !b1 || !W2 || !b2 || !fwd_workspace || !bwd_workspace || !dW_r || !dW1 ||
      !db1 || !dW2 || !db2)
    return SWL_ERR_INVALID_ARG;
  if (T > 0 && (!x || !out || !expert_idx || !gate || !pos_in_expert || !dout || !dx))
    return SWL_ERR_INVALID_ARG;
  if (!std::isfinite(daux)) return SWL_ERR_INVALID_ARG;
  if (!aligned(fwd_workspace, 256) || !aligned(bwd_workspace, 256)) return SWL_ERR_UNSUPPORTED;
  const uintptr_t a = dtype == SWL_BF16 ? 2 : 4;
  if (!aligned(x, a) || !aligned(out, a) || !aligned(dout, a) || !aligned(dx, a) ||
      !aligned(W1, a) || !aligned(W2, a) || !aligned(dW1, a) || !aligned(dW2, a) ||
      !aligned(db1, a) || !aligned(db2, a) || !aligned(W_r, 4) || !aligned(dW_r, 4))
    return SWL_ERR_UNSUPPORTED;
  if (fwd_workspace_bytes < workspace_layout(s, false, 0, nullptr) ||
      bwd_workspace_bytes < backward_workspace_layout(s, 0, nullptr))
    return SWL_ERR_WORKSPACE;
  if (T == 0) return SWL_OK;
  Workspace fw;
  workspace_layout(s, false, reinterpret_cast<uintptr_t>(const_cast<void*>(fwd_workspace)), &fw);
  BwdWorkspace bw;
  backward_workspace_layout(s, reinterpret_cast<uintptr_t>(bwd_workspace), &bw);
  BwdArgs args{x, W_r, b_r, W1, W2, out, expert_idx, gate, pos_in_expert, dout, daux,
               dx, dW_r, db_r, dW1, db1, dW2, db2};
  return launch_backward(s, fw, bw, args, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SWL_OK
             : SWL_ERR_CUDA;
}

swl_status switch_layer_noalloc_status(void* stream) {
  void* scratch = noalloc_scratch_for_current_device();
  if (scratch == nullptr) return SWL_ERR_CUDA;
  return switch_layer_device_status(scratch, stream);   // reads the scratch's header word
}

}  // extern "C"
