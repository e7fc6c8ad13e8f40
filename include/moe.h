/*
 * moe.h -- C ABI of the B200 (sm_100a) DeepSeekMoE layer forward.
 *
 * One MoE layer computes, for every token t,
 *
 *   h_t = x_res_t + sum_{i<Ks} FFN_i(u_t) + sum_{k<K} g_{t,k} FFN_{Ks+idx_{t,k}}(u_t)
 *
 * with SwiGLU experts FFN(v) = W_down (SiLU(W_gate v) * (W_up v)).
 *   - output equation: "DeepSeek Technical Report: MoE Architecture", §1.1(2)
 *     (DeepSeekMoE equation with Ks shared experts), equation [1] of §5.3;
 *   - SwiGLU experts: "DeepSeek-V3 아키텍처 둘러보기", the invariant-core
 *     section (the MLP is SwiGLU);
 *   - gating: §2.3 (softmax gate, DeepSeekMoE / V2) and §3.3 with equations
 *     [3], [4] of §5.3 (sigmoid affinity, bias used for selection only) of
 *     the MoE Architecture report;
 *   - FP8: §3.6 of the same report (E4M3, 1x128 activation tiles, 128x128
 *     weight blocks, fp32 accumulation with promotion every 128 elements).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  T tokens, d hidden, Ks = n_shared, N = n_routed, K = top_k, I = inter,
 *  E = Ks + N experts, R = T*K routed rows.
 *  - All pointers are DEVICE pointers (except `desc`, a host pointer) to
 *    row-major contiguous arrays, 16-byte aligned.  The caller allocates and
 *    owns every buffer, including the workspace; the library allocates
 *    nothing on these paths.
 *  - Shared experts are experts 0..Ks-1 of w_gu / w_down; routed expert j
 *    (0 <= j < N) is expert Ks+j.  topk_idx holds routed indices j.
 *  - w_gu [E, 2I, d]: rows 0..I-1 of an expert are W_gate, rows I..2I-1 W_up.
 *    w_down [E, d, I].
 *  - Every call validates its arguments synchronously and returns a status;
 *    nothing is thrown across the ABI.  Work is enqueued asynchronously on
 *    `stream`.  Problems detected on the device (an index out of range, a
 *    counts array that disagrees with topk_idx, a bounded wait that ran out)
 *    are recorded in a per-device status word read by moe_last_device_status.
 *  - Results are bit-identical from run to run (no floating-point atomics).
 *  - Concurrent calls that share a workspace race; give each stream its own.
 *  - The library cannot see buffer sizes: each buffer must hold at least the
 *    elements its comment states, or a kernel overruns it.
 *  - The kernels of one call are launched with programmatic stream
 *    serialisation and each waits for its predecessor's results before it
 *    touches memory, so stream order is kept as for plain launches.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* a size, pointer, alignment or mode is not accepted */
  MOE_ERR_UNSUPPORTED = 2,   /* valid layer, but a shape the library does not handle */
  MOE_ERR_WORKSPACE = 3,     /* ws_bytes below moe_workspace_size(desc) */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime/driver call or a launch failed */
  MOE_ERR_TIMEOUT = 5,       /* a device-side bounded wait expired (device status) */
  MOE_ERR_DEVICE_CHECK = 6   /* a device-side consistency check failed (device status) */
} moe_status;

typedef enum { MOE_GATE_SOFTMAX = 0, MOE_GATE_SIGMOID = 1 } moe_gate;

typedef enum { MOE_DT_F32 = 0, MOE_DT_BF16 = 1, MOE_DT_E4M3 = 2 } moe_dtype;

/* The layer's problem statement.  Accepted dtype pairs (act_dtype, w_dtype):
 *   (F32, F32)   fp32 activations and weights; GEMMs on tf32 tensor cores,
 *                router in fp32; H, expert outputs and h in fp32.
 *   (BF16, BF16) bf16 activations and weights, fp32 accumulation; H, expert
 *                outputs and h in bf16.
 *   (BF16, E4M3) bf16 x and router (gating stays BF16), E4M3 expert weights
 *                with fp32 128x128 block scales; x and H quantised to E4M3 per
 *                1x128 tile; expert outputs and h in bf16. */
typedef struct moe_layer_desc {
  int32_t T;           /* tokens, >= 0 */
  int32_t d;           /* hidden size */
  int32_t n_shared;    /* Ks >= 0 */
  int32_t n_routed;    /* N, 1..512 */
  int32_t top_k;       /* K, 1..min(N, 16) */
  int32_t inter;       /* I, expert width */
  int32_t gate;        /* moe_gate */
  int32_t renorm;      /* 1: g = s / sum_selected(s); 0: g = s */
  float route_scale;   /* multiplies g after normalisation (1.0; 2.5 for V3) */
  int32_t n_group;     /* expert groups for group-limited routing (1 = none) */
  int32_t topk_group;  /* groups kept; a group's score is the sum of its two largest keys */
  int32_t act_dtype;   /* moe_dtype */
  int32_t w_dtype;     /* moe_dtype */
} moe_layer_desc;

/* Shape rules (MOE_ERR_INVALID_ARG otherwise):
 *   d, I multiples of 64 (bf16), 32 (f32) or 128 (E4M3); I >= 16; d <= 65536;
 *   N % n_group == 0, 1 <= topk_group <= n_group <= 32, N/n_group >= 2 when
 *   n_group > 1, topk_group*(N/n_group) >= K; bias only with sigmoid gating;
 *   R + Ks*T < 2^31. */

/* Bytes of workspace moe_forward needs for `desc` (the other entry points need
 * no more than this).  0 if desc is invalid. */
size_t moe_workspace_size(const moe_layer_desc* desc);

/* (a) Gating.  Router logits l = x W_r^T (fp32 accumulate), affinities s
 * (softmax over the N routed experts, or sigmoid), selection keys s + bias,
 * group limit, top-K with ties to the lower expert index, and gate weights
 * g = route_scale * s (/ sum of the selected s when renorm).  The bias
 * changes the selection only, never g.
 *   x [T, d] act_dtype;  w_router [N, d] act_dtype;  bias [N] fp32 or NULL
 *   topk_idx [T, K] int32 out (ordered by key desc, index asc)
 *   topk_w   [T, K] fp32 out
 *   counts   [N] int32 out (tokens per routed expert) */
moe_status moe_route(const moe_layer_desc* desc, const void* x, const void* w_router,
                     const float* bias, int32_t* topk_idx, float* topk_w, int32_t* counts,
                     void* ws, size_t ws_bytes, cudaStream_t stream);

/* (b) Token -> expert permutation.  offsets = exclusive scan of the counts;
 * the pair (t, k) with expert e = topk_idx[t,k] goes to permuted row
 * slot_of[t*K+k] = offsets[e] + #{t' < t : e in topk_idx[t']} (stable by
 * token), perm_src[row] = t, and x_perm[row] = x[t] (E4M3: the 1x128
 * quantised row and its scales).
 *   counts [N] int32 in: must equal the histogram of topk_idx (checked on the
 *     device; a mismatch or an index outside [0, N) sets MOE_ERR_DEVICE_CHECK)
 *   offsets [N+1], perm_src [R], slot_of [R] int32 out
 *   x_perm  [R, d] act_dtype (F32/BF16), or [R + T, d] E4M3 bytes whose rows
 *     R..R+T-1 hold the quantised x in token order (the shared experts' input)
 *   x_perm_scale [R + T, d/128] fp32 out for E4M3, NULL otherwise
 *   x_perm and x_perm_scale both NULL: only offsets, perm_src and slot_of are
 *     written (x is not read; used by the expert-parallel dispatch below) */
moe_status moe_permute(const moe_layer_desc* desc, const void* x, const int32_t* topk_idx,
                       const int32_t* counts, int32_t* offsets, int32_t* perm_src,
                       int32_t* slot_of, void* x_perm, float* x_perm_scale, void* ws,
                       size_t ws_bytes, cudaStream_t stream);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory: code that runs inside a host framework which owns all device
 * memory and gives an operator no allocator or scratch buffer, or a C caller
 * that only holds the layer's input and output buffers.  The pages have no
 * counterpart; it is a packaging of moe_permute (same arguments minus the
 * workspace, same results bit for bit).
 *   Scratch: a fixed device array of MOE_NOALLOC_HIST_INTS int32 (1 MiB) that
 *   each device that loads this library holds until the process exits.  It
 *   bounds the shape: ceil(T/128) * N <= MOE_NOALLOC_HIST_INTS (T <= 131072
 *   tokens for N = 256); larger shapes return MOE_ERR_UNSUPPORTED with the
 *   reason in moe_last_error_message.  No device memory is allocated or freed.
 *   The first call on a device looks up the array's device address (with that
 *   device current); make that first call before any stream capture.  The
 *   address is kept for the life of the process, so the library does not
 *   support cudaDeviceReset (or another teardown of the primary context)
 *   between calls; the same holds for the per-device set-up of every entry
 *   point.
 *   Every call uses the same array: calls whose work overlaps on the GPU (two
 *   streams, or two host threads) race and must be serialised by the caller.
 *   The array keeps the last call's contents; each call writes every entry it
 *   reads before reading it, so nothing needs clearing. */
#define MOE_NOALLOC_HIST_INTS 262144
moe_status moe_permute_noalloc(const moe_layer_desc* desc, const void* x,
                               const int32_t* topk_idx, const int32_t* counts, int32_t* offsets,
                               int32_t* perm_src, int32_t* slot_of, void* x_perm,
                               float* x_perm_scale, cudaStream_t stream);

/* (c) Shared and routed experts.  One persistent tcgen05 grouped GEMM computes
 * H = SiLU(A W_gate^T) * (A W_up^T) for every expert (A = x for the shared
 * experts, the expert's x_perm rows for routed ones); a second computes
 * Y = H W_down^T and scatters each row, times g_{t,k} (1 for shared experts),
 * to y_slots[t, k] (routed) or y_slots[t, K+s] (shared expert s).
 *   x [T, d] (F32/BF16 shared-expert input; unused for E4M3)
 *   x_perm, x_perm_scale, offsets, slot_of: as written by moe_permute
 *   perm_src: as written by moe_permute (accepted for symmetry; unused)
 *   topk_w [T, K] fp32
 *   w_gu [E, 2I, d], w_down [E, d, I] in w_dtype; for E4M3 their fp32 block
 *     scales w_gu_scale [E, 2I/128, d/128], w_down_scale [E, d/128, I/128]
 *   y_slots [T, K+Ks, d] out: fp32 for F32, bf16 otherwise */
moe_status moe_grouped_swiglu(const moe_layer_desc* desc, const void* x, const void* x_perm,
                              const float* x_perm_scale, const int32_t* offsets,
                              const int32_t* perm_src, const int32_t* slot_of,
                              const float* topk_w, const void* w_gu, const float* w_gu_scale,
                              const void* w_down, const float* w_down_scale, void* y_slots,
                              void* ws, size_t ws_bytes, cudaStream_t stream);

/* (d) Weighted combine and residual: h[t] = x_res[t] + sum_{s<Ks} y[t, K+s]
 * + sum_{k<K} y[t, k], accumulated in fp32 in that order.
 *   x_residual [T, d] act_dtype; y_slots as above; h [T, d] out (fp32 for F32,
 *   bf16 otherwise). */
moe_status moe_combine(const moe_layer_desc* desc, const void* x_residual, const void* y_slots,
                       void* h, cudaStream_t stream);

/* The whole layer: moe_route, moe_permute, moe_grouped_swiglu, moe_combine,
 * with every intermediate in the workspace.
 *   x_residual: NULL means x (pass RMSNorm(u) as x and u as x_residual to
 *     keep the residual outside the normalisation).
 *   topk_idx [T,K], counts [N]: optional int32 copies of the routing result. */
moe_status moe_forward(const moe_layer_desc* desc, const void* x, const void* x_residual,
                       const void* w_router, const float* bias, const void* w_gu,
                       const float* w_gu_scale, const void* w_down, const float* w_down_scale,
                       void* h, int32_t* topk_idx, int32_t* counts, void* ws, size_t ws_bytes,
                       cudaStream_t stream);

/* moe_forward that also keeps the expert pre-activations a = W_gate u and
 * b = W_up u of every active (token, expert) row, rounded to bf16, for
 * moe_backward_saved.  §3.6 of "DeepSeek Technical Report: MoE Architecture"
 * caches the activations the linear layers' backward needs (in FP8 there);
 * here they are kept in the layer's bf16.  bf16 layers only
 * (MOE_ERR_UNSUPPORTED otherwise).
 *   ab_saved [T*K + Ks*T, 2I] bf16 out, moe_saved_ab_bytes(desc) bytes, 16-byte
 *     aligned: row r holds a in columns 0..I-1 and b in I..2I-1.  Rows
 *     0..T*K-1 are the routed pairs in the permuted order of moe_permute
 *     (expert-major, token order inside an expert), then T rows per shared
 *     expert in token order.  The caller owns it; it is only valid together
 *     with the same desc, x, w_router, bias and w_gu.
 * Everything else as moe_forward. */
size_t moe_saved_ab_bytes(const moe_layer_desc* desc);
moe_status moe_forward_save(const moe_layer_desc* desc, const void* x, const void* x_residual,
                            const void* w_router, const float* bias, const void* w_gu,
                            const void* w_down, void* h, int32_t* topk_idx, int32_t* counts,
                            void* ab_saved, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ---- Load balancing (training-time statistics and the bias update) -------
 * "DeepSeek Technical Report: MoE Architecture", §1.2 (L_ExpBal = alpha_1
 * sum_i f_i P_i with f_i the fraction of tokens that chose expert i and P_i
 * the mean routing probability) and §3.3 (auxiliary-loss-free bias update,
 * gamma = 0.001; complementary sequence-wise balance loss). */

/* Affinities s [T, N] fp32 of every token for every routed expert, computed
 * exactly as moe_route computes them (same router GEMM and fp32 softmax or
 * sigmoid; no bias).  ws as for moe_route. */
moe_status moe_route_affinities(const moe_layer_desc* desc, const void* x, const void* w_router,
                                float* s_out, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Per sequence q of seq_len consecutive tokens (seq_len divides T; seq_len = T
 * gives the batch statistics): f_out[q, i] = fraction of the sequence's tokens
 * whose topk_idx holds i, p_out[q, i] = mean of s[t, i] over the sequence.
 * f_out, p_out [T/seq_len, N] fp32.  Deterministic (fixed summation order). */
moe_status moe_balance_stats(const moe_layer_desc* desc, const float* s, const int32_t* topk_idx,
                             int32_t seq_len, float* f_out, float* p_out, cudaStream_t stream);

/* One step of the auxiliary-loss-free rule on the fp32 bias [N], in place:
 * b_i -= gamma when counts[i] is above the mean load T*K/N, b_i += gamma when
 * below, unchanged when equal (the comparison is exact, in integers). */
moe_status moe_bias_update(const moe_layer_desc* desc, const int32_t* counts, float* bias,
                           float gamma, cudaStream_t stream);

/* ---- Expert parallelism ---------------------------------------------------
 * "DeepSeek Technical Report: MoE Architecture" §3.8: the routed experts are
 * split over GPUs; each GPU routes its own tokens, dispatches the permuted rows
 * of every expert to the GPU that holds it, runs the experts it holds on the
 * rows it receives, and returns the results for the combine.  §3.11 adds
 * redundant copies of heavily loaded experts on other GPUs, each copy taking a
 * share of the expert's rows.  The exchange itself (all-to-all of rows) is the
 * caller's collective; these two calls are the compute on either side of it.
 *
 * Expert FFN over caller-given groups of rows: group i (groups[4i..4i+3] =
 * row0, rows, expert, out_row0, device int32) computes, for r < rows,
 *   y_rows[out_row0 + r] = row_w[out_row0 + r] * FFN_expert(x_rows[row0 + r])
 * (row_w NULL: weight 1) with the same GEMMs as moe_grouped_swiglu.  expert
 * indexes w_gu [n_experts, 2I, d] / w_down [n_experts, d, I]; the output
 * ranges of the groups must not overlap.  F32 and BF16 layers
 * (moe_expert_ffn_fp8 below for E4M3).
 *   n_groups 1..1024; x_rows [n_rows_in, d], y_rows [n_rows_out, d], row_w
 *   [n_rows_out] fp32.  A group outside these bounds, or with an expert outside
 *   [0, n_experts), is skipped and sets MOE_ERR_DEVICE_CHECK.
 *   ws: moe_expert_ffn_workspace_size(desc, n_groups, n_rows_out) bytes. */
size_t moe_expert_ffn_workspace_size(const moe_layer_desc* desc, int32_t n_groups,
                                     int32_t n_rows_out);
moe_status moe_expert_ffn(const moe_layer_desc* desc, int32_t n_experts, int32_t n_groups,
                          const int32_t* groups, int32_t n_rows_in, int32_t n_rows_out,
                          const void* x_rows, const float* row_w, const void* w_gu,
                          const void* w_down, void* y_rows, void* ws, size_t ws_bytes,
                          cudaStream_t stream);

/* Dispatch gather: x_rows[row_of[t*K + k]] = x[t] and, when w_rows is not
 * NULL, w_rows[row_of[t*K + k]] = topk_w[t*K + k] -- the send buffer of the
 * exchange, in the row order the caller's plan chose.  x [T, d] act_dtype,
 * topk_w [T, K] fp32, row_of [T*K] int32 (an index outside [0, n_rows) is
 * skipped and sets MOE_ERR_DEVICE_CHECK), x_rows [n_rows, d], w_rows [n_rows]
 * fp32.  F32 and BF16 layers (moe_dispatch_rows_fp8 below for E4M3). */
moe_status moe_dispatch_rows(const moe_layer_desc* desc, const void* x, const float* topk_w,
                             const int32_t* row_of, int32_t n_rows, void* x_rows, float* w_rows,
                             cudaStream_t stream);

/* ---- Expert parallelism over peer memory --------------------------------
 * The exchange of §3.8 written by the compute kernels themselves, with no
 * collective in between: the dispatch gather stores each row straight into
 * the receive buffer of the rank that holds its expert, and the expert FFN's
 * down projection stores each output row straight back into the receive
 * buffer of the rank that sent the row.  The addresses are device addresses
 * of every rank's buffers in this process: other GPUs' memory opened through
 * CUDA IPC (moe_ipc_get_handle on the owner, moe_ipc_open here; NVLink P2P
 * stores), or local buffers.  No kernel waits on another rank: the caller
 * orders the phases (finish the launches, then a barrier over the ranks)
 * between dispatch, expert FFN and combine.
 *
 * moe_dispatch_rows_to: as moe_dispatch_rows, but the send-order row r lands
 * in rank q's buffers, q being the rank with start[q] <= r < start[q+1], at
 * row base[q] + (r - start[q]) of dst->x[q] (row of d act_dtype elements) and
 * of dst->w[q] (the gate weight, fp32; w[q] may be NULL).  start[0] = 0,
 * start[n_ranks] = n_rows, non-decreasing; 1 <= n_ranks <= MOE_MAX_PEERS;
 * x[q] 16-byte aligned wherever rank q receives rows.  For an E4M3 layer the
 * rows are the 1x128-quantised codes (d bytes) and scale[q] receives their
 * tile scales (d/128 fp32 a row; see moe_dispatch_rows_fp8); scale is unused
 * otherwise.  Host struct, read during the call. */
#define MOE_MAX_PEERS 16
typedef struct moe_peer_rows {
  void* x[MOE_MAX_PEERS];
  float* w[MOE_MAX_PEERS];
  float* scale[MOE_MAX_PEERS];
  int32_t start[MOE_MAX_PEERS + 1];
  int32_t base[MOE_MAX_PEERS];
  int32_t n_ranks;
} moe_peer_rows;
moe_status moe_dispatch_rows_to(const moe_layer_desc* desc, const void* x, const float* topk_w,
                                const int32_t* row_of, int32_t n_rows, const moe_peer_rows* dst,
                                cudaStream_t stream);

/* moe_expert_ffn_to: as moe_expert_ffn, but group i's output row r (times
 * row_w[out0 + r], as there) is stored at row r of the buffer at device byte
 * address group_out[i] (uint64 device array [n_groups], 8-byte aligned; each
 * buffer 16-byte aligned and holding the group's rows of d act_dtype
 * elements).  n_rows_out sizes the workspace (H) as in moe_expert_ffn. */
moe_status moe_expert_ffn_to(const moe_layer_desc* desc, int32_t n_experts, int32_t n_groups,
                             const int32_t* groups, int32_t n_rows_in, int32_t n_rows_out,
                             const void* x_rows, const float* row_w, const void* w_gu,
                             const void* w_down, const uint64_t* group_out, void* ws,
                             size_t ws_bytes, cudaStream_t stream);

/* ---- FP8 expert parallelism ("DeepSeek Technical Report: MoE Architecture"
 * §3.6: dispatch in FP8, combine in BF16) -------------------------------------
 * moe_dispatch_rows_fp8: as moe_dispatch_rows for an E4M3 layer: each token's
 * bf16 row is quantised per 1x128 tile (scale = amax/448, codes = E4M3(v *
 * 448/amax), round to nearest even, saturating; the layer's own gather rule)
 * once, and the codes x_rows [n_rows, d] uint8 and tile scales x_rows_scale
 * [n_rows, d/128] fp32 are written to the token's K send rows (with the gate
 * weights to w_rows when not NULL).  moe_dispatch_rows_to does the same for
 * an E4M3 layer, with dst->scale[q] receiving the scales.
 * moe_quantize_rows_fp8: that quantisation of n_rows bf16 rows [n_rows, d]
 * into codes [n_rows, d] and scales [n_rows, d/128] (the shared experts'
 * input on the rank that owns the tokens).
 * moe_expert_ffn_fp8: the layer's FP8 expert GEMMs over caller-given row
 * groups (as moe_expert_ffn): x_rows codes + x_rows_scale in, the expert
 * weights as E4M3 with 128x128 block scales (as moe_forward takes them), H
 * requantised per 1x128 between the GEMMs, bf16 rows out, times row_w.
 * Exactly one of y_rows [n_rows_out, d] bf16 and group_out (per-group output
 * addresses, as moe_expert_ffn_to) is given.  ws:
 * moe_expert_ffn_workspace_size(desc, ...) of the E4M3 layer. */
moe_status moe_dispatch_rows_fp8(const moe_layer_desc* desc, const void* x, const float* topk_w,
                                 const int32_t* row_of, int32_t n_rows, void* x_rows,
                                 float* x_rows_scale, float* w_rows, cudaStream_t stream);
moe_status moe_quantize_rows_fp8(const moe_layer_desc* desc, const void* x, int32_t n_rows,
                                 void* codes, float* scales, cudaStream_t stream);
moe_status moe_expert_ffn_fp8(const moe_layer_desc* desc, int32_t n_experts, int32_t n_groups,
                              const int32_t* groups, int32_t n_rows_in, int32_t n_rows_out,
                              const void* x_rows, const float* x_rows_scale, const float* row_w,
                              const void* w_gu, const float* w_gu_scale, const void* w_down,
                              const float* w_down_scale, void* y_rows, const uint64_t* group_out,
                              void* ws, size_t ws_bytes, cudaStream_t stream);

/* CUDA IPC of device memory (thin wrappers; a handle is MOE_IPC_HANDLE_BYTES
 * opaque bytes).  moe_ipc_get_handle: the handle of the allocation holding
 * dev_ptr and *offset = dev_ptr minus that allocation's base (allocators hand
 * out pieces of larger allocations).  moe_ipc_open: in another process, the
 * device address of that allocation's base (peer access enabled lazily; add
 * the offset); moe_ipc_close unmaps it (pass the base).  CUDA errors return
 * MOE_ERR_CUDA with the message in moe_last_error_message. */
#define MOE_IPC_HANDLE_BYTES 64
moe_status moe_ipc_get_handle(const void* dev_ptr, void* handle, uint64_t* offset);
moe_status moe_ipc_open(const void* handle, void** dev_ptr);
moe_status moe_ipc_close(void* dev_ptr);

/* Combine of returned rows: h[t] = x_res[t] + sum_{s<Ks} y_shared[s*T + t]
 * + sum_{k<K} y_rows[row_of[t*K + k]], in fp32, in that order (the order of
 * moe_combine, so with the same row values the two agree bit for bit).
 *   y_shared [Ks*T, d] (NULL when Ks = 0), y_rows [n_rows, d], row_of [T*K]
 *   int32; an index outside [0, n_rows) is skipped and sets
 *   MOE_ERR_DEVICE_CHECK.  Element types as for moe_combine. */
moe_status moe_combine_rows(const moe_layer_desc* desc, const void* x_residual,
                            const void* y_shared, const void* y_rows, const int32_t* row_of,
                            int32_t n_rows, void* h, cudaStream_t stream);

/* ---- Layer backward (bf16) ------------------------------------------------
 * The gradients of the layer for an upstream gradient dh = dL/dh, by the
 * chain rule of the output equation above through SwiGLU experts, the gate
 * weights and the affinities ("DeepSeek Technical Report: MoE Architecture",
 * §1.1(2) and equation [1] of §5.3 for the output, §2.3 and §3.3 with
 * equations [3]/[4] of §5.3 for the gating; §3.6 lists the activation- and
 * weight-backward GEMMs of every linear layer).  Per active (token, expert)
 * row with gate weight g (1 for shared experts): a = W_gate u, b = W_up u,
 * z = SiLU(a) b, dz = g W_down^T dh, da = dz b SiLU'(a), db = dz SiLU(a),
 * du += W_gate^T da + W_up^T db, dW_down += g dh z^T, dW_gate += da u^T,
 * dW_up += db u^T, dg = <dh, W_down z>; then the gate-weight backward
 * (renorm: ds_k = c (dg_k - sum_k' dg_k' s_k' / S) / S), the affinity backward
 * (sigmoid: dl = ds s (1 - s); softmax: dl = s (ds - <ds, s>)), and the
 * router: du += W_r^T dl, dW_r = dl^T u.  No gradient flows through the
 * selection, and the selection bias gets none.  The residual's gradient is dh
 * itself and is not written.
 * The call recomputes the routing, the permutation and the pre-activations
 * a, b from x (nothing is kept from the forward).  bf16 layers only
 * (MOE_ERR_UNSUPPORTED otherwise); N*2 bytes must be a multiple of 16.
 *   x [T, d], w_router [N, d], w_gu [E, 2I, d], w_down [E, d, I], dh [T, d]: bf16 in
 *   bias [N] fp32 or NULL (selection only, as in moe_route)
 *   dx [T, d] bf16 out: gradient of x through the experts and the router
 *   dw_router [N, d] fp32 out; dw_gu [E, 2I, d] fp32 out; dw_down [E, d, I]
 *     fp32 out (overwritten, zeros for experts no token reaches)
 *   ws: moe_backward_workspace_size(desc) bytes. */
size_t moe_backward_workspace_size(const moe_layer_desc* desc);
moe_status moe_backward(const moe_layer_desc* desc, const void* x, const void* w_router,
                        const float* bias, const void* w_gu, const void* w_down, const void* dh,
                        void* dx, float* dw_router, float* dw_gu, float* dw_down, void* ws,
                        size_t ws_bytes, cudaStream_t stream);

/* moe_backward with the three weight gradients written as bf16 (rounded to
 * nearest even from the fp32 accumulators) instead of fp32: §3.6 of the same
 * report keeps weight gradients in BF16 (master weights and optimizer maths in
 * FP32).  dw_router [N, d], dw_gu [E, 2I, d], dw_down [E, d, I] bf16 out;
 * everything else as moe_backward. */
moe_status moe_backward_bf16_grads(const moe_layer_desc* desc, const void* x,
                                   const void* w_router, const float* bias, const void* w_gu,
                                   const void* w_down, const void* dh, void* dx, void* dw_router,
                                   void* dw_gu, void* dw_down, void* ws, size_t ws_bytes,
                                   cudaStream_t stream);

/* The backward from the pre-activations moe_forward_save kept, instead of
 * recomputing them: the gate/up GEMM of the recomputation (a quarter of the
 * backward's tensor-core work) is skipped; routing and the permutation are
 * still rebuilt from x, which yields the same rows because both are
 * deterministic.  ab_saved as written by moe_forward_save with the same desc,
 * x, w_router, bias and w_gu (not checked); bf16_grads nonzero: dw_router,
 * dw_gu and dw_down bf16 as in moe_backward_bf16_grads, else fp32 as in
 * moe_backward.  Launches moe_backward_launch_count(desc) - 1 kernels.
 * Everything else, workspace included, as moe_backward. */
moe_status moe_backward_saved(const moe_layer_desc* desc, const void* x, const void* w_router,
                              const float* bias, const void* w_gu, const void* w_down,
                              const void* dh, const void* ab_saved, void* dx, void* dw_router,
                              void* dw_gu, void* dw_down, int32_t bf16_grads, void* ws,
                              size_t ws_bytes, cudaStream_t stream);

/* ---- The backward with FP8 GEMMs (E4M3 layers) ----------------------------
 * "DeepSeek Technical Report: MoE Architecture", §3.6: the activation-backward
 * and weight-backward GEMMs in FP8 E4M3, activations per 1x128 tile, weights
 * per 128x128 block, fp32 accumulation promoted every 128 elements; gating in
 * BF16; weight gradients in BF16.  Same gradients as moe_backward.
 * Tiles run along the dimension each GEMM contracts over: x and dh rows (over
 * d) for a, b = W_gate u, W_up u and dz' = W_down^T dh; the [da | db] rows
 * (over 2I) for du; and, for dW_down = sum dh (g z)^T and dW_gu = sum
 * [da | db] u^T, which contract over an expert's rows, tiles of 128 rows x 1
 * column, the expert's rows taken in token order and padded with zero rows to
 * a multiple of 128 (a shared expert's rows are all T tokens).
 * Weights: E4M3 codes and 128x128 block scales as the forward's
 * (moe_quantize_fp8_blockwise), and of the transposed matrices
 * (moe_quantize_fp8_blockwise_t): every GEMM reads its weight K-major, so
 * W_gate/W_up serve the recomputed a, b as they are and du transposed, and
 * W_down serves dz' = W_down^T dh transposed only,
 *   w_gu [E, 2I, d] + w_gu_scale [E, 2I/128, d/128],
 *   w_gu_t [E, d, 2I] + w_gu_t_scale [E, d/128, 2I/128],
 *   w_down_t [E, I, d] + w_down_t_scale [E, I/128, d/128]
 * (the transposed codes and scales of the forward's, since a block's amax
 * does not depend on its orientation).
 *   x [T, d] bf16, w_router [N, d] bf16, bias [N] fp32 or NULL, dh [T, d] bf16
 *   dx [T, d] bf16 out; dw_router [N, d], dw_gu [E, 2I, d], dw_down [E, d, I]
 *     bf16 out (zeros for experts no token reaches)
 *   ws: moe_backward_fp8_workspace_size(desc) bytes (0 for non-E4M3 layers).
 * E4M3 layers only, with d a multiple of 256, K + Ks <= 32 and N*2 a multiple
 * of 16 (MOE_ERR_UNSUPPORTED otherwise); tensors 16-byte aligned, scales
 * 4-byte aligned.  Launches moe_backward_fp8_launch_count(desc) kernels. */
size_t moe_backward_fp8_workspace_size(const moe_layer_desc* desc);
moe_status moe_backward_fp8(const moe_layer_desc* desc, const void* x, const void* w_router,
                            const float* bias, const void* w_gu, const float* w_gu_scale,
                            const void* w_gu_t, const float* w_gu_t_scale, const void* w_down_t,
                            const float* w_down_t_scale, const void* dh, void* dx,
                            void* dw_router, void* dw_gu, void* dw_down, void* ws,
                            size_t ws_bytes, cudaStream_t stream);
int32_t moe_backward_fp8_launch_count(const moe_layer_desc* desc);

/* Number of kernels moe_backward launches for `desc` (0 if invalid or T = 0). */
int32_t moe_backward_launch_count(const moe_layer_desc* desc);

/* Offline FP8 quantisation of weights in 128x128 blocks (not on the hot path).
 * w_bf16 [batch, rows, cols] bf16 in; w_e4m3 [batch, rows, cols] bytes out;
 * scale [batch, rows/128, cols/128] fp32 out.  rows, cols multiples of 128.
 * Rule per block: amax = max|w|, scale = amax/448, code = E4M3_rn_satfinite(
 * w * (448/amax)) in fp32; an all-zero block gets scale 0 and zero codes. */
moe_status moe_quantize_fp8_blockwise(const void* w_bf16, int32_t rows, int32_t cols,
                                      int32_t batch, void* w_e4m3, float* scale,
                                      cudaStream_t stream);

/* moe_quantize_fp8_blockwise of the transposed matrices, without forming
 * them: w_e4m3_t [batch, cols, rows] codes and scale_t [batch, cols/128,
 * rows/128] (the transposed layout of the same codes and scales, a 128x128
 * block's amax being the same either way).  The transposed weights of
 * moe_backward_fp8.  Same arguments and errors otherwise. */
moe_status moe_quantize_fp8_blockwise_t(const void* w_bf16, int32_t rows, int32_t cols,
                                        int32_t batch, void* w_e4m3_t, float* scale_t,
                                        cudaStream_t stream);

/* Human-readable name of a status. */
const char* moe_status_string(moe_status status);

/* Synchronises `stream`, then returns and clears the current device's status
 * word (MOE_OK if no device-side check fired since the last call). */
moe_status moe_last_device_status(cudaStream_t stream);

/* Stage timing.  While set on the calling host thread, moe_forward records
 * events[0] before routing, [1] after routing, [2] after the permutation,
 * [3] after the gate/up GEMM, [4] after the down GEMM and [5] after the
 * combine, on the call's stream; moe_grouped_swiglu records [2], [3] and [4]
 * around its own launches.  n must be 6 (events owned by the caller); pass
 * NULL, 0 to stop. */
moe_status moe_trace_events(cudaEvent_t* events, int32_t n);

/* Text describing the last MOE_ERR_CUDA returned on the calling host thread
 * (the failing call and the CUDA error name); "" if none.  Owned by the
 * library, valid until the next call on this thread. */
const char* moe_last_error_message(void);

/* Number of kernels moe_forward launches for `desc` (0 if invalid). */
int32_t moe_forward_launch_count(const moe_layer_desc* desc);

/* Self-test of the device-side bounded wait: launches one block that waits on
 * a shared-memory barrier nothing ever completes, gives up after limit_us
 * microseconds (1..1000000), records MOE_ERR_TIMEOUT in the status word and
 * returns.  The context stays usable. */
moe_status moe_selftest_bounded_wait(uint32_t limit_us, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
