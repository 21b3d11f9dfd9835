/*
 * switch_layer.h -- C ABI of a B200 (sm_100a) implementation of the forward
 * pass of one Switch Transformer expert layer.
 *
 * The layer (sources: "Switch Transformer" reading note, eightmm.github.io,
 * sections "Router", "Expert FFN Layer", "Capacity Factor", "Load-Balancing
 * Loss"; paper-graph summary of arXiv 2101.03961 "Switch Transformers: Scaling
 * to Trillion Parameter Models with Simple and Efficient Sparsity", section 3.4:
 * "The mathematics of routing", "The loss formulation", the expert-capacity
 * formula, "The routing mechanics in detail", "The selective precision
 * solution"; "Switch Transformer, explained." recipe steps 2-5):
 *
 *   z_t   = W_r x_t + b_r                     router logits, fp32 (bf16 layers: computed
 *                                             on the tensor cores from the exact split
 *                                             W_r = hi + mid + lo into three bf16
 *                                             matrices, products exact, fp32 accumulation)
 *   p_t   = softmax(z_t)                      fp32
 *   e_t   = argmax_i p_t,i                    lowest index on ties
 *   g_t   = p_t,e_t                           gate
 *   C     = ceil(capacity_factor * T / N)     expert capacity
 *   pos_t = #{ s < t : e_s = e_t }            0-based position in token order
 *   kept  = pos_t < C                         overflow tokens are dropped
 *   out_t = kept ? g_t * (W2[e] relu(W1[e] x_t + b1[e]) + b2[e]) : 0
 *   aux   = N * sum_i f_i * P_i,  f_i = #{t : e_t = i} / T,  P_i = mean_t p_t,i
 *
 * No residual is added (a dropped token's layer output is zero; the caller's
 * residual connection carries it).  aux is returned without the alpha factor.
 *
 * Conventions for every entry point:
 *  - Memory: every tensor pointer is a DEVICE pointer owned by the caller
 *    (except the *_host arguments of switch_layer_forward_host_io, which are
 *    host pointers, ideally pinned).  The library allocates nothing and keeps no
 *    state between calls besides a launch counter and the fixed scratch array of
 *    switch_layer_forward_noalloc.
 *  - Layouts: contiguous row-major.  x [T,d]; W_r [N,d] fp32; b_r [N] fp32;
 *    W1 [N,d_ff,d]; b1 [N,d_ff]; W2 [N,d,d_ff]; b2 [N,d]; out [T,d];
 *    expert_idx, pos_in_expert [T] int32; gate [T] fp32; aux_loss [1] fp32.
 *    x, W1, b1, W2, b2 and out share the activation dtype (SWL_F32 or SWL_BF16).
 *  - Asynchrony: calls enqueue work on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and return; outputs are valid once the stream has
 *    executed the work.  Device-side failures are read with
 *    switch_layer_device_status.
 *  - Errors: arguments are validated on the host before anything is enqueued;
 *    an invalid call returns a non-zero swl_status and enqueues nothing.
 *    Nothing traps or aborts.
 *  - Thread safety: calls may be made from several host threads; two calls that
 *    share a workspace must not overlap on the GPU.
 */
#ifndef SWITCH_LAYER_H
#define SWITCH_LAYER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SWL_ABI_VERSION 1

typedef enum swl_status {
  SWL_OK = 0,
  SWL_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad dtype or capacity factor */
  SWL_ERR_UNSUPPORTED = 2,  /* valid but not handled: bf16 with d or d_ff not a multiple of 8,
                               misaligned pointer, sizes beyond int32 indexing */
  SWL_ERR_WORKSPACE = 3,    /* workspace smaller than switch_layer_workspace_size() */
  SWL_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, copy, event) */
  SWL_ERR_DEVICE = 5        /* a kernel reported a failure (see switch_layer_device_status) */
} swl_status;

typedef enum swl_dtype { SWL_F32 = 0, SWL_BF16 = 1 } swl_dtype;

/* Workspace flag: also reserve device staging buffers for switch_layer_forward_host_io. */
#define SWL_WS_HOST_IO 1
/* Workspace flag: size for switch_layer_forward_top2 (not combinable with SWL_WS_HOST_IO). */
#define SWL_WS_TOP2 2
/* Workspace flag: size for switch_layer_forward_ntlb (not combinable with the others). */
#define SWL_WS_NTLB 4

/* Number of timed stages and their order (see switch_layer_forward_timed):
 * 0 router (logits; for N <= 128 also softmax/argmax/ranks; bf16 layers include
 * the split of W_r into its bf16 pieces), 1 router softmax for N > 128 (empty
 * otherwise), 2 dispatch scan + aux loss, 3 dispatch gather, 4 expert FFN
 * (GEMM1 + bias + ReLU and GEMM2 + bias + gate + combine).  For N <= 128 and
 * batches whose x is at most 16 MiB, scan and gather run as one kernel, timed in
 * stage 2; stage 3 is then empty. */
#define SWL_NUM_STAGES 5

/* Expert capacity C = ceil(capacity_factor * T / N) ("Capacity Factor" section
 * of the reading note), evaluated exactly on the binary value of the double
 * capacity_factor.  Returns -1 for T < 0, N <= 0 or a capacity factor that is
 * not finite and positive; saturates at INT64_MAX. */
int64_t switch_layer_capacity(int64_t T, int64_t N, double capacity_factor);

/* Device workspace bytes needed by a forward call of this shape (flags: 0,
 * SWL_WS_HOST_IO, SWL_WS_TOP2 or SWL_WS_NTLB).  The workspace must be 256-byte aligned; its contents need
 * no initialisation.  Returns SWL_ERR_INVALID_ARG / SWL_ERR_UNSUPPORTED for
 * shapes the forward call would reject. */
swl_status switch_layer_workspace_size(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                       double capacity_factor, int flags, size_t* bytes);

/* Forward pass of the Switch layer (formulas above).
 *   T, d, d_ff, N   tokens, model width, expert FFN width, experts (T = 0 is an
 *                   empty batch: nothing is written except *aux_loss = 0)
 *   dtype           SWL_F32 or SWL_BF16: dtype of x, W1, b1, W2, b2, out
 *   x ... b2        inputs (layouts above); W_r and b_r are always fp32
 *   capacity_factor > 0, finite
 *   out             [T,d] layer output (zero rows for dropped tokens)
 *   expert_idx      [T] e_t
 *   gate            [T] g_t = p_t,e_t (fp32)
 *   pos_in_expert   [T] pos_t; the token was dropped iff pos_t >= C
 *   aux_loss        [1] N * sum_i f_i P_i (f before the capacity cut)
 *   b_r             [N] router-logit bias or NULL for none
 *   workspace       device scratch of workspace_bytes >= switch_layer_workspace_size()
 *   stream          cudaStream_t to enqueue on
 * bf16 additionally requires d % 8 == 0, d_ff % 8 == 0 and 16-byte aligned x,
 * W1, W2, out and W_r (TMA rows, vector loads); otherwise SWL_ERR_UNSUPPORTED. */
swl_status switch_layer_forward(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                const void* x, const float* W_r, const void* W1, const void* b1,
                                const void* W2, const void* b2, double capacity_factor,
                                void* out, int32_t* expert_idx, float* gate,
                                int32_t* pos_in_expert, float* aux_loss, const float* b_r,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Top-2 variant: the earlier-MoE routing the pages compare the Switch layer
 * with ("Switch Transformer" reading note, "Comparison to Earlier MoE":
 * y_t = sum over the two largest p_t,i of p_t,i E_i(x_t); the attention-and-MoE
 * note's example normalises the two weights within the selected set).
 *   e_t,0 = argmax_i p_t,i, e_t,1 = argmax over i != e_t,0 (lowest index on ties)
 *   g_t,k = p_t,e_t,k, divided by (p_t,e_t,0 + p_t,e_t,1) when normalize = 1
 *   C     = ceil(2 * capacity_factor * T / N)  (capacity grows with k: paper-graph
 *           summary, "Expert capacity can be at least halved")
 *   pos_t,k = assignments to e_t,k by tokens before t (token order; a token's two
 *           experts differ); assignment (t, k) is dropped iff pos_t,k >= C
 *   out_t = sum over kept k of g_t,k E_e_t,k(x_t)   (zero if both are dropped)
 *   aux   = N * sum_i f_i P_i with f_i counting FIRST choices (the loss
 *           formula's argmax indicator)
 * expert_idx, gate and pos_in_expert are [T, 2] (row-major: first choice,
 * second choice).  Requires 2 <= N <= 2048 (SWL_ERR_INVALID_ARG /
 * SWL_ERR_UNSUPPORTED) and a workspace sized with SWL_WS_TOP2; normalize is 0
 * or 1.  Other arguments, layouts and errors as switch_layer_forward. */
swl_status switch_layer_forward_top2(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                     const void* x, const float* W_r, const void* W1,
                                     const void* b1, const void* W2, const void* b2,
                                     double capacity_factor, int normalize, void* out,
                                     int32_t* expert_idx, float* gate, int32_t* pos_in_expert,
                                     float* aux_loss, const float* b_r, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* No-Token-Left-Behind variant (paper-graph summary of arXiv 2101.03961,
 * Appendix B, in the capacity-factor discussion: tokens that overflow their
 * first expert are rerouted to their second-choice expert, a two-stage process;
 * the paper reports no benefit from it).  The readings taken:
 *   e_t,0, e_t,1  first and second choice as in switch_layer_forward_top2;
 *                 g_t,k = p_t,e_t,k (unnormalised)
 *   C             = ceil(capacity_factor * T / N), one slot per token (top-1)
 *   stage 1       pos_t,0 = first choices of e_t,0 by tokens before t (the top-1
 *                 position); the token is kept there iff pos_t,0 < C
 *   stage 2       for a token stage 1 dropped, in token order:
 *                 pos_t,1 = min(c_e, C) + (earlier tokens stage 1 dropped whose
 *                 second choice is e = e_t,1), c_e = first choices of e;
 *                 kept at e_t,1 iff pos_t,1 < C; pos_t,1 = -1 for a token stage 1 kept
 *   out_t         = g_t,k E_e_t,k(x_t) for the stage k that keeps it, else 0
 *   aux           = N * sum_i f_i P_i with f_i counting first choices
 * expert_idx, gate and pos_in_expert are [T, 2] (row-major).  Requires
 * 2 <= N <= 2048, ReLU experts and a workspace sized with SWL_WS_NTLB; other
 * arguments, layouts and errors as switch_layer_forward. */
swl_status switch_layer_forward_ntlb(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                     const void* x, const float* W_r, const void* W1,
                                     const void* b1, const void* W2, const void* b2,
                                     double capacity_factor, void* out, int32_t* expert_idx,
                                     float* gate, int32_t* pos_in_expert, float* aux_loss,
                                     const float* b_r, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* Backward pass of switch_layer_forward (top-1 routing, ReLU experts): the
 * gradients of L = sum(dout * out) + daux * aux_loss.  The router's gradient
 * flows through the gate only ("Switch Transformer, explained", "Why one expert
 * is enough": the chosen expert's output is scaled by its router probability)
 * and through P_i of the aux loss, f_i being a count without gradient
 * (paper-graph summary, "The loss formulation"); argmax, positions and the
 * capacity cut pass no gradient.  For a kept token t of expert e, gate g,
 * h = relu(W1[e] x + b1[e]), u = W2[e] h + b2[e]:
 *   du = g dout_t, dW2[e] += du h^T, db2[e] += du,
 *   da = (W2[e]^T du) * [h > 0], dW1[e] += da x^T, db1[e] += da, dx_t += W1[e]^T da,
 *   dg_t = dout_t . u (computed as (dout_t . out_t) / g from the bf16 output);
 * for every token, with p_t = softmax(W_r x_t + b_r) recomputed in fp32:
 *   dz_t,j = dg_t g (delta_{j e} - p_t,j) [kept] + daux (N / T) p_t,j (f_j - sum_i f_i p_t,i)
 *   dW_r = sum_t dz_t x_t^T, db_r = sum_t dz_t, dx_t += W_r^T dz_t.
 * Arguments: the forward's inputs and outputs (out, expert_idx, gate,
 * pos_in_expert) and its workspace, unchanged since that call (the packed
 * expert inputs, hidden rows and expert bases are read from it); dout [T, d]
 * (activation dtype), daux (host value); outputs dx [T, d], dW1, db1, dW2, db2
 * in the activation dtype and the weights' layouts, dW_r [N, d] and db_r [N]
 * fp32 (db_r may be NULL).  bwd_workspace: switch_layer_backward_workspace_size
 * bytes, 256-byte aligned.  Every output is written (experts without kept
 * tokens get zero gradients).  Errors as switch_layer_forward. */
swl_status switch_layer_backward_workspace_size(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                                int dtype, double capacity_factor,
                                                size_t* bytes);
swl_status switch_layer_backward(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                 const void* x, const float* W_r, const float* b_r,
                                 const void* W1, const void* b1, const void* W2, const void* b2,
                                 double capacity_factor, const void* out,
                                 const int32_t* expert_idx, const float* gate,
                                 const int32_t* pos_in_expert, const void* fwd_workspace,
                                 size_t fwd_workspace_bytes, const void* dout, float daux,
                                 void* dx, float* dW_r, float* db_r, void* dW1, void* db1,
                                 void* dW2, void* db2, void* bwd_workspace,
                                 size_t bwd_workspace_bytes, void* stream);

/* Layer variants the pages name beside the Switch layer, in one call:
 *   top_k = 2     the top-2 routing of switch_layer_forward_top2 (routing outputs
 *                 [T, 2]), with normalize as there;
 *   activation    SWL_ACT_RELU (the Switch expert) or SWL_ACT_GEGLU: the paper-graph
 *                 summary's "ReLU or GEGLU" expert, read as
 *                 E(x) = W2 (GELU(W_g x + b_g) * (W_v x + b_v)) + b2 with the exact
 *                 GELU(u) = u Phi(u); W1 is then [N, 2 d_ff, d] (W_g rows, then W_v
 *                 rows) and b1 [N, 2 d_ff] (b_g, then b_v);
 *   router_noise  NULL (inference), or [T, d] fp32 multiplicative noise on the
 *                 router input ("input jitter", Table 11 of the paper-graph
 *                 summary, a training-time exploration): the router sees x * noise
 *                 in fp32 (bf16 layers: split exactly into three bf16 pieces for
 *                 the tensor-core logits kernel at any N; fp32 layers and
 *                 SWL_ROUTER_FFMA: the FFMA router), the experts see x.
 * A NULL variant is switch_layer_forward.  The workspace is sized by
 * switch_layer_variant_workspace_size with the same variant (only whether
 * router_noise is NULL matters there).  Invalid fields: SWL_ERR_INVALID_ARG. */
#define SWL_ACT_RELU 0
#define SWL_ACT_GEGLU 1
typedef struct swl_variant {
  int top_k;
  int normalize;
  int activation;
  const float* router_noise;
} swl_variant;
swl_status switch_layer_variant_workspace_size(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                               int dtype, double capacity_factor,
                                               const swl_variant* variant, size_t* bytes);
swl_status switch_layer_forward_variant(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                        int dtype, const void* x, const float* W_r,
                                        const void* W1, const void* b1, const void* W2,
                                        const void* b2, double capacity_factor, void* out,
                                        int32_t* expert_idx, float* gate,
                                        int32_t* pos_in_expert, float* aux_loss,
                                        const float* b_r, const swl_variant* variant,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* As switch_layer_forward, and records cudaEvent_t stage_events[k] on `stream`
 * before stage 0 (k = 0) and after stage k-1 (k = 1..SWL_NUM_STAGES): an array
 * of SWL_NUM_STAGES + 1 events created by the caller (timing enabled). */
swl_status switch_layer_forward_timed(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                      const void* x, const float* W_r, const void* W1,
                                      const void* b1, const void* W2, const void* b2,
                                      double capacity_factor, void* out, int32_t* expert_idx,
                                      float* gate, int32_t* pos_in_expert, float* aux_loss,
                                      const float* b_r, void* workspace, size_t workspace_bytes,
                                      void* stream, void* const* stage_events);

/* End-to-end variant with HOST input and outputs: copies x_host to the device,
 * runs the forward pass, and copies out, expert_idx, gate, pos_in_expert and
 * aux_loss back into the *_host buffers, all enqueued on `stream` (the caller
 * synchronises the stream before reading them).  Weights stay device pointers.
 * The workspace must be sized with SWL_WS_HOST_IO; it holds the device copies. */
swl_status switch_layer_forward_host_io(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                        const void* x_host, const float* W_r, const void* W1,
                                        const void* b1, const void* W2, const void* b2,
                                        double capacity_factor, void* out_host,
                                        int32_t* expert_idx_host, float* gate_host,
                                        int32_t* pos_in_expert_host, float* aux_loss_host,
                                        const float* b_r, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* Synchronises `stream` and returns the device status of the last forward call
 * that used `workspace`: SWL_OK, or SWL_ERR_DEVICE if a kernel reported a
 * failure (a bounded pipeline wait expired, or non-finite router logits).
 * SWL_ERR_CUDA if the synchronisation itself failed. */
swl_status switch_layer_device_status(const void* workspace, void* stream);

/* ---- One global batch sharded over ranks by contiguous token ranges ----
 *
 * Data parallelism over the tokens of ONE batch: rank g of `world` ranks holds
 * the g-th contiguous range of the batch's T_total tokens (rank order = token
 * order) and a full copy of the weights.  Positions, the capacity cut and the
 * aux loss are those of the unsharded batch: a token's position is the number
 * of tokens of its expert on earlier ranks plus its position among this rank's
 * tokens (the cumulative sum over the expert's column of the dispatch mask in
 * token order, "The routing mechanics in detail"), C = ceil(cf * T_total / N),
 * and f_i, P_i count the whole batch ("The loss formulation").  One exchange is
 * needed: every rank's per-expert token counts and sums of p.  A forward pass is
 * three steps on every rank:
 *   1. switch_layer_forward_shard_begin: routing of the local tokens, and this
 *      rank's exchange record (switch_layer_shard_record_bytes(N) bytes, a
 *      multiple of 16: N int32 token counts, then N fp64 sums of p at the next
 *      16-byte boundary);
 *   2. the caller gathers the records of all ranks, in rank order, into one
 *      device buffer of world * record bytes (an all-gather: NCCL
 *      ncclAllGather, torch.distributed.all_gather_into_tensor);
 *   3. switch_layer_forward_shard_end: offsets of earlier ranks, the capacity
 *      cut, the aux loss (the same value on every rank), dispatch and the expert
 *      FFN of the local kept tokens.
 * Both calls take the local T and the same workspace (sized by
 * switch_layer_workspace_size for the local T); expert_idx, gate and
 * pos_in_expert written by step 1 are read and completed by step 3 (pos_in_expert
 * holds in-block ranks in between and the global position after).  A record set
 * whose counts do not add up to T_total, or to this rank's T, makes the device
 * status SWL_ERR_DEVICE.  With world = 1 the result equals switch_layer_forward's. */

/* Bytes of one rank's exchange record for N experts (0 for invalid N). */
size_t switch_layer_shard_record_bytes(int64_t N);

/* Step 1 of a sharded forward (see above).  T: this rank's tokens (may be 0),
 * T_total >= T: tokens of the whole batch; x, W_r, b_r, expert_idx, gate,
 * pos_in_expert as for switch_layer_forward; record: device, 16-byte aligned,
 * switch_layer_shard_record_bytes(N) bytes, written by the call. */
swl_status switch_layer_forward_shard_begin(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                            int dtype, int64_t T_total, const void* x,
                                            const float* W_r, const float* b_r,
                                            double capacity_factor, int32_t* expert_idx,
                                            float* gate, int32_t* pos_in_expert, void* record,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream);

/* Step 3 of a sharded forward.  rank in [0, world); gathered: device, 16-byte
 * aligned, the world records in rank order; the remaining arguments as for
 * switch_layer_forward, with the tensors of step 1. */
swl_status switch_layer_forward_shard_end(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                          int dtype, int64_t T_total, int rank, int world,
                                          const void* gathered, const void* x, const void* W1,
                                          const void* b1, const void* W2, const void* b2,
                                          double capacity_factor, void* out,
                                          int32_t* expert_idx, float* gate,
                                          int32_t* pos_in_expert, float* aux_loss,
                                          void* workspace, size_t workspace_bytes, void* stream);

/* ---- Expert parallelism over ranks (experts sharded, tokens sharded) ----
 *
 * The pages' multi-device design: every device hosts a subset of the experts,
 * and tokens travel to the device of their expert and back in an all-to-all
 * (paper-graph summary, "The routing mechanics in detail": dispatch, expert
 * computation, output recombination; "Switch Transformer, explained", recipe
 * step 4).  Rank r of `world` ranks (N % world == 0) holds the weights of
 * experts [r L, r L + L), L = N / world, as W1_local [L, d_ff, d], b1_local
 * [L, d_ff], W2_local [L, d, d_ff], b2_local [L, d], the full router W_r, and
 * the r-th contiguous token range of one global batch of T_total tokens.  The
 * result is the unsharded layer's: the same positions, capacity cut, aux loss
 * and outputs.  A forward pass on every rank:
 *   1. switch_layer_forward_shard_begin (routing, exchange record);
 *   2. all-gather of the records (as for the global-batch split), and a host
 *      copy of them for the all-to-all sizes: switch_layer_ep_counts gives, per
 *      peer, the rows this rank sends and receives (kept tokens only);
 *   3. switch_layer_ep_dispatch: positions and aux loss from the records, and
 *      this rank's kept token rows packed into send_rows [sum send, d] in the
 *      order peer, expert, position;
 *   4. all-to-all: peer g's block of send_rows goes to peer g (NCCL
 *      ncclSend/ncclRecv or torch.distributed.all_to_all_single with the counts
 *      of step 2), arriving in recv_rows [sum recv, d] in source-rank order;
 *   5. switch_layer_ep_experts: the received rows of this rank's experts through
 *      their FFN (bias, no gate), written back in the receive order into
 *      ret_rows [sum recv, d];
 *   6. the reverse all-to-all (recv counts become send counts) into
 *      back_rows [sum send, d];
 *   7. switch_layer_ep_combine: out_t = g_t * (the token's returned row), or 0
 *      for a dropped token.
 * Every rank's workspace is sized by switch_layer_ep_workspace_size (its own
 * tokens plus room for L * min(C, T_total) received rows:
 * switch_layer_ep_max_recv_rows).  Row buffers are device memory in the
 * activation dtype, 16-byte aligned for bf16. */
int64_t switch_layer_ep_max_recv_rows(int64_t N, int world, int64_t T_total,
                                      double capacity_factor);
swl_status switch_layer_ep_workspace_size(int64_t T, int64_t d, int64_t d_ff, int64_t N,
                                          int dtype, int world, int64_t T_total,
                                          double capacity_factor, size_t* bytes);
/* Host-only: rows this rank sends to (send_rows[g]) and receives from
 * (recv_rows[g]) every peer g, from a host copy of the gathered records. */
swl_status switch_layer_ep_counts(int64_t N, int world, int rank, int64_t T_total,
                                  double capacity_factor, const void* gathered_host,
                                  int64_t* send_rows, int64_t* recv_rows);
swl_status switch_layer_ep_dispatch(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                    int world, int rank, int64_t T_total,
                                    double capacity_factor, const void* gathered, const void* x,
                                    int32_t* expert_idx, int32_t* pos_in_expert,
                                    float* aux_loss, void* send_rows, void* workspace,
                                    size_t workspace_bytes, void* stream);
/* n_recv: rows in recv_rows (the sum of recv counts); ret_rows holds as many. */
swl_status switch_layer_ep_experts(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                   int world, int rank, int64_t T_total, double capacity_factor,
                                   const void* gathered, void* recv_rows, int64_t n_recv,
                                   const void* W1_local, const void* b1_local,
                                   const void* W2_local, const void* b2_local, void* ret_rows,
                                   void* workspace, size_t workspace_bytes, void* stream);
swl_status switch_layer_ep_combine(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                   int world, int rank, int64_t T_total,
                                   double capacity_factor, const void* back_rows,
                                   const int32_t* expert_idx, const float* gate,
                                   const int32_t* pos_in_expert, void* out, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Bytes of the fixed device scratch used by switch_layer_forward_noalloc. */
#define SWL_NOALLOC_MAX_BYTES (64u << 20)

/* Forward pass for callers that cannot call cudaMalloc: plugin code running
 * inside a host framework that owns all device memory and forbids allocations
 * outside its own allocator, and latency-critical loops where an allocation (a
 * synchronising, device-wide call) is not acceptable.  The paper has no
 * counterpart of this entry point: it is switch_layer_forward
 * with the workspace taken from a fixed-size static device array inside this
 * library (SWL_NOALLOC_MAX_BYTES, held by every GPU that loads the library until
 * the process exits).  Inputs and outputs are still passed by the caller, with
 * the same meaning, layouts and checks as switch_layer_forward.
 *  - Shapes whose workspace (switch_layer_workspace_size with flags 0) exceeds
 *    SWL_NOALLOC_MAX_BYTES are rejected with SWL_ERR_WORKSPACE before anything
 *    is enqueued.
 *  - The first call on a device looks up the device address of the static
 *    array for the current device (which must be the device of `stream`); make
 *    that first call before any stream capture.
 *  - All calls on a device share the one array, and it keeps the contents of the
 *    last call; the call re-initialises what must start at zero.  Calls that
 *    overlap on the GPU (different streams, or host threads without ordering)
 *    race on the array and give wrong results: serialise them.
 *  - The device address of the array is looked up once per device and kept
 *    for the life of the process: after cudaDeviceReset (which unloads the
 *    library's device code) this entry point and switch_layer_noalloc_status
 *    must not be called again on that device.
 *  - Device-side failures of this variant are read with
 *    switch_layer_noalloc_status (switch_layer_device_status needs a workspace
 *    pointer, which this variant has none of).
 *  - Allocates nothing: no cudaMalloc / cudaFree or allocating library call. */
swl_status switch_layer_forward_noalloc(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                        const void* x, const float* W_r, const void* W1,
                                        const void* b1, const void* W2, const void* b2,
                                        double capacity_factor, void* out, int32_t* expert_idx,
                                        float* gate, int32_t* pos_in_expert, float* aux_loss,
                                        const float* b_r, void* stream);

/* Synchronises `stream` and returns the device status of the last
 * switch_layer_forward_noalloc call on the current device: SWL_OK, or
 * SWL_ERR_DEVICE if one of its kernels reported a failure (a bounded pipeline
 * wait expired, or non-finite router logits); SWL_ERR_CUDA if the
 * synchronisation or the read failed.  Like the entry point it reports on, it
 * allocates nothing.  The paper has no counterpart of this call either. */
swl_status switch_layer_noalloc_status(void* stream);

/* Human-readable name of a status code (static string). */
const char* switch_layer_status_string(swl_status status);

/* Name of timed stage k (0 <= k < SWL_NUM_STAGES), or NULL. */
const char* switch_layer_stage_name(int k);

/* Number of kernel launches this library has issued since it was loaded. */
uint64_t switch_layer_launch_count(void);

/* How the fp32 router logits of bf16 layers are computed (process-wide; fp32
 * layers always use FFMA).  Both give the float32 dot product up to the rounding
 * of fp32 accumulation ("The selective precision solution"):
 *   SWL_ROUTER_TENSOR (default): tcgen05 tensor cores on the exact split of
 *     W_r into three bf16 pieces (hi + mid + lo), fp32 accumulation in TMEM;
 *   SWL_ROUTER_FFMA: fp32 FMA on the CUDA cores, no tensor cores.
 * The choice changes the workspace size: set it before
 * switch_layer_workspace_size and keep it for the calls that use that
 * workspace.  Returns SWL_ERR_INVALID_ARG for an unknown mode. */
typedef enum swl_router_mode { SWL_ROUTER_TENSOR = 0, SWL_ROUTER_FFMA = 1 } swl_router_mode;
swl_status switch_layer_set_router_mode(int mode);
int switch_layer_router_mode(void);

/* ---- Failure-path test hooks (process-wide; not for production use) ----
 * Every wait inside the kernels (pipeline barriers, the expert FFN's wait for
 * another CTA's hidden rows) gives up after a time limit, sets the device
 * status to SWL_ERR_DEVICE and lets the kernel drain and return, so the CUDA
 * context stays usable.  switch_layer_set_wait_limit_ns sets that limit (0
 * restores the default of 2 s).  switch_layer_set_stall_test(1) makes the
 * expert FFN wait for one GEMM1 epilogue warp more than token tile 0 has, a
 * signal that never comes: the wait runs out after the limit and the call
 * reports SWL_ERR_DEVICE through switch_layer_device_status (outputs of that
 * call are undefined).  switch_layer_set_stall_test(0) (the default) turns it
 * off; other values return SWL_ERR_INVALID_ARG. */
swl_status switch_layer_set_wait_limit_ns(uint64_t ns);
swl_status switch_layer_set_stall_test(int on);

/* The kernels switch_layer_forward would launch for this shape on a GPU of
 * num_sms SMs, under the current router mode, without touching the device
 * (host-only; usable without a GPU).  Writes a NUL-terminated list of
 * comma-separated key=value pairs into the caller's buffer buf of len bytes:
 *   router            tc | tc_wide (tensor-core router: fused for N <= 128 /
 *                     logits only for N > 128, top-2 or a jittered input) |
 *                     ffma_warpsplit | ffma_tile | ffma_wide
 *   ksplit            CTAs per router tile (cluster size) or K slices
 *   router_stages     operand stages per tensor-core router CTA (0: FFMA router)
 *   softmax           fused (in the router, N <= 128) | stream (N > 128, one
 *                     logits slice, N % 4 == 0, N <= 2048: bulk-copied row
 *                     chunks) | rows (row in registers) | wide (three passes)
 *   tokens_per_block  tokens per router block (the dispatch's unit)
 *   dispatch          fused (scan and gather in one launch) | two_kernel
 *   ffn               sm100 (bf16, tcgen05) | f32 (SIMT)
 *   tile_rows         token rows per expert GEMM tile
 *   accumulators      TMEM accumulators of the bf16 expert FFN (0 for f32)
 * Returns SWL_OK, the shape's validation error (as switch_layer_workspace_size),
 * or SWL_ERR_INVALID_ARG when buf is NULL, num_sms <= 0 or len is too small
 * (256 bytes always suffice). */
swl_status switch_layer_describe_plan(int64_t T, int64_t d, int64_t d_ff, int64_t N, int dtype,
                                      double capacity_factor, int num_sms, char* buf,
                                      size_t len);

#ifdef __cplusplus
}
#endif

#endif /* SWITCH_LAYER_H */
