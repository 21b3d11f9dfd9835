// Internal interface between the C-ABI host code (switch_layer.cu) and the
// kernels of the Switch-layer forward.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace swl {

// Device error word values (first int of the workspace header).
enum DeviceError : int {
  kDevOk = 0,
  kDevPipelineTimeout = 1,   // a GEMM pipeline wait exceeded its time limit
  kDevIndexOutOfRange = 2,   // an index check failed (should never happen)
  kDevNonFiniteLogits = 3,   // a token had no finite maximum logit (NaN/Inf input)
};

constexpr int kTokensPerBlock = 256;   // largest token block of the softmax / rank / gather stages
constexpr int kMaxExperts = 1 << 20;

// Workspace header (256 bytes at offset 0).
struct WsHeader {
  int err;                  // DeviceError of the last call
  unsigned int done;        // arrival counter of the dispatch-scan kernel (self-resetting)
  unsigned int next_tile;   // work counter of the expert FFN kernel (zeroed by the scan)
  int gather_prefetch;      // set by the scan: at least half of the tokens are kept, so
                            // the gather reads every row before its destination is known
  int pad[60];
};

// Device pointers carved out of the caller's workspace.
struct Workspace {
  WsHeader* hdr;
  float* logits;        // [ksplit_eff, T, N] fp32 partial logits (slice 0 reused for p)
  int* blk_count;       // [nblk, N] assignments of block b's tokens to expert e
  int* blk_count1;      // top-2: [nblk, N] first choices of block b's tokens for e
  int* blk_off;         // [nblk, N] tokens of earlier blocks routed to e
  float* blk_psum;      // [nblk, N] sum over block b of p_{t,e}
  int* exp_count;       // [N] assignments to e (tokens whose argmax is e for top-1)
  int* exp_count1;      // top-2: [N] tokens whose first choice is e
  int* exp_rows;        // [N] kept rows m_e = min(count_e, C)
  int* exp_base;        // [N] first packed row of expert e
  int* exp_off;         // [N] shard of a global batch: tokens of e on earlier ranks
  int* tile_prefix;     // [N+1] prefix over experts of ceil(m_e / tile_rows)
  double* psum64;       // [N] sum over all tokens of p_{t,e}
  int* slot_token;      // [A] packed row -> assignment (token t, choice k: t * topk + k)
  int* ready;           // [T/16 + N + 1] per token tile: GEMM1 epilogue warps done
  int* tile_prefix2;    // GEMM2 split: [N+1] tile prefix counting split sub-tiles
  int* split_base;      // GEMM2 split: [N] first partial-tile group of e, -1: not split
  float* part;          // GEMM2 split: [kSplitMaxGroups][split][tile_rows][128] fp32
  int* split_grp;       // GEMM2 split: [kSplitMaxGroups][4] (expert, m-tile, token tile,
                        // 0) of each group, expert -1 past the last group
  int* split_ready;     // GEMM2 split: [kSplitMaxGroups][kSplitFactor] per split token tile
                        // and K chunk: GEMM1 epilogue warps done (zeroed by the scan)
  void* w3;             // tensor-core router: [3N, d] bf16 pieces hi, mid, lo of W_r
  float* xj;            // jittered router input x * noise [T, d] fp32 (jitter on the FFMA router)
  void* x3;             // jittered router input as three bf16 pieces [3T, d] (xsplit)
  void* xbuf;           // [A, d] packed expert inputs (act dtype), A = T * topk
  void* hbuf;           // [A, d_ff] packed hidden activations (act dtype)
  void* ybuf;           // top-2: [A, d] gated expert output per assignment (act dtype)
  int* ntlb_rank2;      // No-Token-Left-Behind: [T] in-block rank of an overflow token
                        // among the block's overflow tokens with the same second choice
  float* ntlb_gate;     // No-Token-Left-Behind: [T] router probability of the keeping expert
  void* ntlb_rec;       // No-Token-Left-Behind: per-expert totals scratch of the two scans
  // host-I/O staging (only with SWL_WS_HOST_IO)
  void* x_dev;
  void* out_dev;
  int* idx_dev;
  float* gate_dev;
  int* pos_dev;
  float* aux_dev;
  size_t total_bytes;
};

struct Shape {
  int64_t T, d, d_ff, N;
  int dtype;      // 0 = fp32, 1 = bf16
  int64_t C;      // capacity (formula value, from the batch's T_total tokens)
  int64_t C_eff;  // min(C, T): rows an expert can actually keep on this rank
  int64_t T_total;  // tokens of the whole batch (T unless a shard of a global batch)
  int64_t C_cmp;  // min(C, T_total): a token is kept iff its position is below it
  int sharded;    // 1: a shard of a global batch (positions offset by earlier ranks)
  int ffn_split;  // GEMM2 split over K of experts with full token tiles (1: none)
  int topk;       // experts per token: 1 (Switch) or 2 (the top-2 variant)
  int glu;        // 1: GEGLU experts (W1 [N, 2 d_ff, d]: gate rows, then value rows)
  int jitter;     // 1: the router sees x * noise (a jittered fp32 copy of x)
  int xsplit;     // jitter on the tensor-core logits (wide bf16 layers): the fp32 router
                  // input is split exactly into three bf16 pieces like W_r
  int normalize;  // top-2: gates divided by their sum
  int ntlb;       // 1: No-Token-Left-Behind (top-2 router, one slot per token, capacity of
                  // top-1; tokens stage 1 drops go to their second choice's free slots)
  int router_path;  // RouterPath
  int tpb;        // tokens per block of the softmax / rank / gather stages (<= kTokensPerBlock)
  int nblk;       // ceil(T / tpb)
  int kslice;     // K elements per slice of the router logits GEMM (multiple of 16)
  int ksplit_eff; // K slices of the router logits GEMM (partials summed by the softmax)
  int tile_rows;  // token rows per GEMM tile (N of the UMMA, or the SIMT tile)
};

// Router kernel choice for a shape (a pure function of the shape).
enum RouterPath : int {
  kRouterWarpSplit = 0,   // N <= 128, small T: one CTA per 2048/BN tokens, K split over warps
  kRouterTile = 1,        // N <= 128, large T: 256x64 / 128x128 tiles, whole K per CTA
  kRouterWide = 2,        // N > 128: logits GEMM (K slices) + softmax kernel
  kRouterTC = 3,          // bf16 layers, N <= 128: tcgen05 logits from a 3-piece bf16 split
                          // of W_r, 128-token tiles, K split over a cluster of 1/2/4 CTAs
  kRouterTCWide = 4,      // bf16 layers, N > 128: tcgen05 logits tiles (128 x 128) to the
                          // workspace, then the softmax kernel
};
struct RouterPlan {
  int path;     // RouterPath
  int tpb;      // tokens per dispatch block
  int kslice;   // K per logits slice (wide, tile and tensor-core paths)
  int ksplit;   // logits slices (CTAs of a cluster on the tile / tensor-core paths)
};
// tensor != 0: the tensor-core router (bf16 layers); else the FFMA kernels.
RouterPlan router_plan(int64_t T, int64_t d, int64_t N, int tensor, int topk = 1,
                       int force_wide = 0);

size_t workspace_layout(const Shape& s, bool host_io, uintptr_t base, Workspace* ws);

// Packed expert rows an FFN call may fill: one per assignment (T * topk), one per
// token for No-Token-Left-Behind.
inline int64_t packed_rows(const Shape& s) { return s.T * (s.ntlb ? 1 : s.topk); }

// ---- stage launchers (all asynchronous on `stream`; return cudaGetLastError()).
// N <= kFusedRouterMaxN: one fused kernel (logits + softmax + block statistics);
// launch_router_softmax is then not called.  Wider N: logits here, softmax after.
constexpr int kFusedRouterMaxN = 128;
// Jittered router input: ws.xj = x * noise (fp32, element by element).
cudaError_t launch_router_jitter(const Shape& s, const Workspace& ws, const void* x,
                                 const float* noise, cudaStream_t stream);
cudaError_t launch_router_logits(const Shape& s, const Workspace& ws, const void* x,
                                 const float* W_r, const float* b_r, int* expert_idx, float* gate,
                                 int* local_rank, cudaStream_t stream);
// Tensor-core router (kRouterTC, kRouterTCWide): splits W_r into ws.w3, then routes.
// tmX = x as bf16 [T, d] (box 64 x 128), tmW = ws.w3 as bf16 [3N, d] (box 64 x
// router_tc_padded_experts(N)), both with 128-byte swizzle.  Two launches.  The
// router CTAs also prefetch [l2_prefetch, +l2_prefetch_bytes) into L2 once their
// own loads have landed (16-byte aligned, a multiple of 16 bytes; 0 bytes: none).
int router_tc_padded_experts(int64_t N);
// Pipeline stages of the tensor-core router kernel for this shape on a GPU of
// num_sms SMs (what launch_router_tc uses).
int router_tc_stages(const Shape& s, int num_sms);
cudaError_t launch_router_tc(const Shape& s, const Workspace& ws, const float* W_r,
                             const CUtensorMap& tmX, const CUtensorMap& tmW, const float* b_r,
                             int* expert_idx, float* gate, int* local_rank,
                             const void* l2_prefetch, size_t l2_prefetch_bytes, int num_sms,
                             cudaStream_t stream);
// Expert weights fetched into L2 during the router and dispatch stages.
constexpr size_t kL2PrefetchBytes = 64u << 20;
// Softmax kernel of a shape: none (fused into the router, N <= 128), the
// streaming kernel (one logits slice, N % 4 == 0, N <= kStreamSoftmaxMaxN), the
// register-row kernel (N <= 2048) or the three-pass kernel (any N).
enum SoftmaxVariant : int { kSoftmaxFused = 0, kSoftmaxStream = 1, kSoftmaxRows = 2,
                            kSoftmaxWide = 3 };
constexpr int kStreamSoftmaxMaxN = 2048;
int softmax_variant(const Shape& s);
cudaError_t launch_router_softmax(const Shape& s, const Workspace& ws, const float* b_r,
                                  int* expert_idx, float* gate, int* local_rank,
                                  cudaStream_t stream);
// GEMM2 split over K (see expert_gemm_sm100.cu): at most kSplitMaxGroups groups
// (an expert's 128-feature by token-tile GEMM2 tile) are split per call.
constexpr int kSplitMaxGroups = 128;
constexpr int kSplitFactor = 4;
struct SplitPlan {
  int factor;        // 1: no split
  int m_tiles2;      // GEMM2 feature tiles (d / 128)
  int max_groups;
  int* tile_prefix2;
  int* split_base;
  int* groups;       // [max_groups][4]
  int* ready;        // [max_groups][kSplitFactor] chunk readiness counters, zeroed here
};
// record != nullptr: a shard of a global batch; the expert totals go to the
// exchange record and the expert-level part waits for launch_shard_combine.
cudaError_t launch_dispatch_scan(const Shape& s, const Workspace& ws, float* aux_loss,
                                 void* record, cudaStream_t stream);
// No-Token-Left-Behind (s.ntlb): the two stages' positions, kept rows and aux
// loss (after the top-2 router), then the gather of the kept tokens' rows.
cudaError_t launch_ntlb_positions(const Shape& s, const Workspace& ws, const int* expert_idx,
                                  int* pos_in_expert, float* aux_loss, cudaStream_t stream);
cudaError_t launch_ntlb_gather(const Shape& s, const Workspace& ws, const void* x,
                               const int* expert_idx, const float* gate, int* pos_in_expert,
                               void* out, cudaStream_t stream);
// Exchange record of one rank: int32 counts [N], then fp64 sums of p [N] at a
// 16-byte aligned offset.
size_t shard_record_psum_offset(int64_t N);
size_t shard_record_bytes(int64_t N);
// Offsets of earlier ranks, kept rows, bases, tile prefix and the global aux
// loss from the records of all `world` ranks (gathered in rank order).
cudaError_t launch_shard_combine(const Shape& s, const Workspace& ws, const void* gathered,
                                 int rank, int world, float* aux_loss, cudaStream_t stream);
cudaError_t launch_dispatch_gather(const Shape& s, const Workspace& ws, const void* x,
                                   const int* expert_idx, int* pos_in_expert, void* out,
                                   cudaStream_t stream);
// Expert parallelism: where the owner rank's received rows go (see
// ep_plan_kernel in dispatch.cu).  The arrays live in the owner's workspace.
struct EpPlan {
  int64_t N;        // experts of the layer
  int world, rank;  // ranks; this rank owns experts [rank L, rank L + L)
  int L;            // experts per rank
  int64_t C_cmp;    // min(C, T_total)
  int64_t max_rows; // rows of the owner's packed buffers: L * C_cmp
  int tile_rows;
  int* blk_src;     // [world L] first receive row of block (source g, local expert l)
  int* blk_dst;     // [world L] its first packed row
  int* blk_n;       // [world L] its rows
  int* rows;        // [L] kept rows of each local expert (all sources)
  int* base;        // [L] first packed row of each local expert
  int* tile_prefix; // [L + 1]
  int* ready;       // [max_rows / 16 + L + 1]
  WsHeader* hdr;
};
cudaError_t launch_ep_plan(const EpPlan& ep, const void* gathered, cudaStream_t stream);
// dir 0: receive order -> packed buffer; dir 1: packed buffer -> receive order.
cudaError_t launch_ep_permute(const EpPlan& ep, void* recv, void* packed, int64_t n_recv,
                              int row_bytes, int dir, cudaStream_t stream);
// Source side: out[t] = gate * returned row (kept) or 0 (dropped).
cudaError_t launch_ep_combine(const Shape& s, const Workspace& ws, const void* ret,
                              const int* expert_idx, const float* gate,
                              const int* pos_in_expert, void* out, cudaStream_t stream);
// Top-2: out[t] = sum over the token's kept assignments of their gated rows.
cudaError_t launch_combine_top2(const Shape& s, const Workspace& ws, const int* pos_in_expert,
                                void* out, cudaStream_t stream);
// Scan and gather in one launch, for N <= 128 and small batches (one CTA per
// router block copies its tokens' rows; the two-kernel path spreads large copies
// over more warps).
bool dispatch_fused_ok(const Shape& s);
cudaError_t launch_dispatch_fused(const Shape& s, const Workspace& ws, const void* x,
                                  const int* expert_idx, int* pos_in_expert, void* out,
                                  float* aux_loss, cudaStream_t stream);
// Both expert GEMMs (bf16, tcgen05) in one persistent launch: GEMM1 + bias + ReLU
// into hbuf, GEMM2 + bias + gate scattered to out (gate == nullptr: GEMM2 +
// bias written to the packed rows of out, for the expert-parallel path).
cudaError_t launch_expert_ffn_bf16(const Shape& s, const Workspace& ws, const CUtensorMap& tmA1,
                                   const CUtensorMap& tmB1, const CUtensorMap& tmA2,
                                   const CUtensorMap& tmB2, const void* b1, const void* b2,
                                   const float* gate, void* out, int num_sms,
                                   cudaStream_t stream);
cudaError_t launch_expert_gemm_f32(const Shape& s, const Workspace& ws, int which,
                                   const void* W, const void* bias, const float* gate, void* out,
                                   cudaStream_t stream);

// ---- backward pass (backward.cu)
struct BwdWorkspace {
  float* dg;          // [T] gradient of each token's gate (0 for dropped tokens)
  int* counts;        // [N] argmax counts (f = counts / T)
  int* tile_prefix;   // [N + 1] 64-row tiles of packed rows per expert
  float* dz;          // [T, N] gradient of the router logits
  void* du;           // [T, d] packed rows g * dout (act dtype)
  void* da;           // [T, d_ff] packed rows of the gradient of the pre-activations
  float* dx_acc;      // [T, d] fp32 accumulator of dx
  float* part;        // split partials of the column sums and of the router's dW_r
};
struct BwdArgs {
  const void* x;          // [T, d]
  const float* W_r;       // [N, d]
  const float* b_r;       // [N] or null
  const void* W1;         // [N, d_ff, d]
  const void* W2;         // [N, d, d_ff]
  const void* out;        // [T, d] forward output
  const int* expert_idx;
  const float* gate;
  const int* pos_in_expert;
  const void* dout;       // [T, d]
  float daux;
  void* dx;               // [T, d]
  float* dW_r;            // [N, d]
  float* db_r;            // [N] or null
  void* dW1;              // [N, d_ff, d]
  void* db1;              // [N, d_ff]
  void* dW2;              // [N, d, d_ff]
  void* db2;              // [N, d]
};
size_t backward_workspace_layout(const Shape& s, uintptr_t base, BwdWorkspace* w);
cudaError_t launch_backward(const Shape& s, const Workspace& fw, const BwdWorkspace& bw,
                            const BwdArgs& a, cudaStream_t stream);

// Tile rows for the bf16 tcgen05 GEMMs given the effective capacity.
int bf16_tile_rows(int64_t C_eff);
// TMEM accumulators of the bf16 expert FFN for a token tile of tile_rows rows:
// four of 128 columns when the tile fits 128, else two of 256 (the rule the FFN
// launcher applies to its 512 TMEM columns).
inline int ffn_accumulators(int tile_rows) { return tile_rows <= 128 ? 4 : 2; }
constexpr int kF32TileRows = 32;

// Number of kernel launches issued by this library since load.
void count_launch(int n = 1);
// Bound of every wait inside the kernels, in ns (switch_layer_set_wait_limit_ns).
unsigned long long wait_limit_ns();
// Failure-path test of the expert FFN (switch_layer_set_stall_test).
bool stall_test_enabled();

#ifdef __CUDACC__
// Range check of a computed index.  In a checked build (-DSWL_CHECKED) a failed
// check records kDevIndexOutOfRange in the device error word and returns false,
// and the caller skips the access; other builds compile it to `true`.
__device__ __forceinline__ bool checked_index(bool ok, int* err) {
#ifdef SWL_CHECKED
  if (!ok) atomicExch(err, kDevIndexOutOfRange);
  return ok;
#else
  (void)ok;
  (void)err;
  return true;
#endif
}
#endif

// Programmatic dependent launch: a kernel launched with launch_dependent() may
// start while the previous kernel on the stream is still finishing; it must call
// pdl_wait() before touching memory that kernel reads or writes.  Every kernel
// calls pdl_trigger() early so that its dependent can be scheduled.
#ifdef __CUDACC__
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
#endif

}  // namespace swl
