/*
 * moe_b200.h - C ABI of the B200 (sm_100a) routed + shared-expert MoE layer.
 *
 * One MoE layer forward = five calls, in this order on the caller's streams:
 *
 *   main stream:  moe_router_topk -> moe_align_sort -> moe_stage1_gemm
 *                 -> moe_stage2_gemm_accumulate (waits on the addend event)
 *   side stream:  shared_expert_gate_dot -> moe_stage1_gemm (identity routing)
 *                 -> moe_stage2_gemm_accumulate (identity routing, writes the
 *                    addend) -> record the addend event
 *
 * Sources (web pages; the section named is where the operation is stated):
 *   [65207] vllm-project/vllm PR 65207, "Purpose": commit 1 folds
 *           routed_scaling_factor into the top-k weights inside
 *           biased_grouped_topk; commit 2 hands the shared-expert output to the
 *           routed experts as the stage-2 addend plus a ready event, the
 *           aux-stream shared expert overlapping sorting and stage 1, the
 *           stage-2 GEMM epilogue accumulating it; "Dependencies": the
 *           capability is feature-detected (supports_output_addend).
 *           Reviewer measurements, "Commits 2 and 3": moe_sorting without
 *           zeroing the output.
 *   [6106]  ROCm/aiter PR 6106 "[Triton/Gluon] Add per token scale to a8w8 moe
 *           gemm", "Technical Details": x_token_scale (fp32, one per row of x)
 *           and w_expt_scale (fp32, one per expert) multiply the fp32
 *           accumulator in the epilogue before activation and fused quant;
 *           rows follow the gather index; MXFP8 uses BLOCK_K = 32, K % 32 == 0.
 *   [56789] vllm-project/vllm PR 56789 (shared_expert_gate as a tiny dot),
 *           "Summary" and "Commits": sigmoid(x . w_gate) as one fp32-
 *           accumulated dot with the sigmoid folded in; the output is stored in
 *           the input dtype so the store does the rounding.
 *
 * Conventions, all calls:
 *   - Tensor pointers are DEVICE pointers owned by the caller. The calls
 *     allocate no memory. Every call is asynchronous on the given stream.
 *   - Arguments are checked on the host first; on any invalid argument the
 *     call returns a negative status and launches nothing.
 *   - MOE_ERR_CUDA: a CUDA runtime call failed; moe_last_cuda_error() gives
 *     the message (per thread).
 *   - Kernels never trap: a device-side check or a bounded wait that gives up
 *     records a code in a device error word read by moe_device_error().
 *   - Layouts are row-major and dense unless stated. T tokens, H hidden, E
 *     routed experts, k = top_k, I expert intermediate size.
 *   - With MOE_B200_PAIR=1 in the environment, the grouped GEMMs of 16- and
 *     128-token blocks run on CTA pairs (2-CTA clusters sharing one M = 256
 *     tensor-core MMA, each SM loading its 128 weight rows and half of the
 *     token rows) when the weight rows split into an even number of 128-row
 *     tiles (stage 1: I % 128 == 0, except the fp8 stage 1, whose per-row
 *     quantisation follows a grid barrier; stage 2: H % 256 == 0); by default
 *     one CTA per tile (measured faster on every workload but fp8 decode).
 *     Results do not depend on the choice.
 *   - Shapes the grouped GEMMs cover (anything else returns MOE_ERR_SHAPE or
 *     MOE_ERR_ALIGNMENT and launches nothing): H % 128 == 0 (stage 1 with bf16
 *     operands: H % 64 == 0), I % 64 == 0, and I % 128 == 0 for MXFP8 and
 *     MXFP4; token blocks (block_m) of 16, 32, 64, 128 or 256 rows (at most
 *     128 for MXFP8 / MXFP4). Smaller alignments (H % 16, block_m = 8) are
 *     not supported.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* CUDA handles are passed as opaque pointers (cudaStream_t / cudaEvent_t). */
typedef void* moe_stream_t;
typedef void* moe_event_t;

typedef int moe_status_t;
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)       /* null pointer, out-of-range size or mode */
#define MOE_ERR_UNSUPPORTED_DTYPE (-2) /* dtype not accepted by this call */
#define MOE_ERR_ALIGNMENT (-3)         /* pointer not 16-byte aligned, K % 32 != 0 for MXFP8 */
#define MOE_ERR_SHAPE (-4)             /* sizes the kernels do not cover */
#define MOE_ERR_CUDA (-5)              /* a CUDA runtime / driver call failed */
#define MOE_ERR_DEVICE (-6)            /* device error word was set (moe_device_error) */
#define MOE_ERR_WORKSPACE_LIMIT (-7)   /* problem larger than the library's static workspace */

/* Operand formats. */
#define MOE_DT_BF16 0
#define MOE_DT_FP16 1
#define MOE_DT_FP8_E4M3 2   /* e4m3 codes; fp32 scale per token row of x, per expert of W [6106] */
#define MOE_DT_MXFP8_E4M3 3 /* e4m3 codes; ue8m0 byte per 32 K elements of every row [6106] */
#define MOE_DT_F32 4
/* MXFP4 weights against MXFP8 activations (stage 1 and stage 2 only): W13 and
 * W2 hold OCP e2m1 codes, two per byte (element 2j in bits 0-3 of byte j,
 * element 2j+1 in bits 4-7), one ue8m0 byte per 32 K elements of every row,
 * packed by moe_mx_pack_weight_scales as for MXFP8; x, h and their scales are
 * exactly the MXFP8 operands. The pages run MXFP4 checkpoints on this layer
 * ([65207] commit 3: Quark OCP MX MoE method); they fix no activation format,
 * and MXFP8 keeps the stage-2 operand h at 8 bits. */
#define MOE_DT_MXFP4_E2M1 5

/* Routing modes of moe_router_topk. */
#define MOE_ROUTE_SOFTMAX 0
#define MOE_ROUTE_GROUPED_SIGMOID 1

/* Largest sizes the kernels cover. */
#define MOE_MAX_EXPERTS 512
#define MOE_MAX_TOPK 32

/* ------------------------------------------------------------------------ */

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status_t status);
/* Library version string. */
const char* moe_version(void);
/* Message of the last failed CUDA call made by this thread inside the library. */
const char* moe_last_cuda_error(void);
/* 1: moe_stage2_gemm_accumulate accepts an output addend and a ready event
 * (the capability query of [65207] "Dependencies"). */
int moe_supports_output_addend(void);

/* Reads the current device's error word into *code (0 = none) and clears it.
 * Synchronises `stream` first. Codes: 1 = bounded mbarrier wait gave up,
 * 2 = expert id out of range in the sort, 3 = sorted slot id out of range,
 * 4 = a block_expert entry outside [0, E) met by a grouped GEMM (the block is
 * then computed with expert 0's weights, so no access leaves the weights). */
moe_status_t moe_device_error(int* code, moe_stream_t stream);

/* Self-test of the failure path: launches one CTA whose thread waits, through
 * the grouped GEMM's own bounded mbarrier wait, on a barrier phase that nothing
 * completes. After the wait limit (4 s) it records device error 1 and returns;
 * the context stays usable. Read the code with moe_device_error. Asynchronous
 * on `stream`. */
moe_status_t moe_selftest_wait_timeout(moe_stream_t stream);

/* Number of int32 slots the padded sort output may need: T*top_k +
 * E*(block_m - 1) rounded up to a multiple of block_m ("capacity rows").
 * sorted_ids holds this many entries, block_expert this / block_m, and the
 * stage-1 output h this many rows. */
size_t moe_sorted_capacity(int T, int top_k, int E, int block_m);

/* Bytes of the fp32 accumulation workspace of moe_stage2_gemm_accumulate:
 * T*H floats followed by T*ceil(H/128) int32 arrival counters. The caller
 * zeroes it ONCE after allocating it; each complete call leaves it zeroed. */
size_t moe_stage2_workspace_bytes(int T, int H);

/* Bytes of the stage-1 workspace for `dtype` (0 for invalid arguments), for
 * `capacity` rows; 256-byte aligned parts, in this order:
 *  - MOE_DT_FP8_E4M3: the unquantised h as fp32 [rows, I], a per-tile row
 *    amax and one arrival counter per token block;
 *  - the token rows of x copied into sorted order [rows, H] (x's element
 *    type), which the GEMM then reads with one TMA box per 128-byte K atom
 *    (identity routing reads x itself and leaves this part unused);
 *  - MOE_DT_MXFP8_E4M3 / MOE_DT_MXFP4_E2M1: the token scale bytes placed in
 *    512-byte tiles, one per (token block, 128 columns of H).
 * The caller zeroes it ONCE after allocating it; each complete call leaves the
 * counters at zero. */
size_t moe_stage1_workspace_bytes(int dtype, int T, int top_k, int E, int H, int I, int block_m);

/* Bytes of the packed block-scale tiles of one projection's weights (MXFP8 or
 * MXFP4: one ue8m0 byte per 32 K elements either way): which = 0 for W13
 * ([E,2I,H] weights), which = 1 for W2 ([E,H,I] weights). 0 unless H and I are
 * multiples of 128. */
size_t moe_mx_weight_scale_bytes(int which, int E, int H, int I);

/* Bytes of the MXFP8 scale tiles of the stage-1 output h (capacity rows of I
 * columns); 0 for an unsupported shape. */
size_t moe_mx_h_scale_bytes(int T, int top_k, int E, int I, int block_m);

/* moe_mx_pack_weight_scales: one-off weight preparation for MXFP8 and MXFP4
 * weights (no counterpart on the pages; MXFP8 itself is [6106]'s BLOCK_K = 32
 * format, and MXFP4 weights carry the same one-byte scale per 32 elements).
 * src holds the ue8m0 scale bytes row-major, [E, rows, K/32] (which = 0: W13,
 * rows = 2I, K = H; which = 1: W2, rows = H, K = I). dst
 * (moe_mx_weight_scale_bytes) receives them as 512-byte tiles, one per
 * (expert, 128-row weight tile, 128-column K stage): byte (m % 32)*16 +
 * (m / 32)*4 + b holds the scale of tile row m and K block b. For W13 the tile
 * rows are ordered as the stage-1 kernel reads them: tile row m = rr + 16*gu +
 * 32*qq is W13 row gu*I + (4*tile + qq)*16 + rr (16 gate rows, then their 16
 * up rows). Checks: H % 128 == 0, I % 128 == 0. Asynchronous on `stream`. */
moe_status_t moe_mx_pack_weight_scales(int which, const void* src, void* dst, int E, int H, int I,
                                       moe_stream_t stream);

/* ------------------------------------------------------------------------ */

/* moe_router_topk: top-k routing of T tokens over E experts.
 * [65207] "Purpose", commit 1: routed_scaling_factor is applied inside this
 * call, to the top-k weights, instead of to the layer output.
 *
 *   logits          fp32 [T,E]   router logits (the model's gate linear).
 *   correction_bias fp32 [E] or NULL (GROUPED_SIGMOID only; NULL = 0).
 *   mode MOE_ROUTE_SOFTMAX: pick the k largest logits (ties: lower index);
 *        weights exp(l_j - m)/sum_sel exp(l_i - m) (renormalize != 0) or the
 *        full softmax at the picked experts (renormalize == 0).
 *   mode MOE_ROUTE_GROUPED_SIGMOID: s = fp32(sigmoid(l)) evaluated in double;
 *        c = s + bias (fp32); group score = sum of the two largest c of each
 *        of n_group equal groups; keep topk_group groups (ties: lower group);
 *        pick k experts of the kept groups by c (ties: lower index); weights
 *        s_j / sum_sel s (renormalize != 0) or s_j.
 *   Both modes multiply the weights by routed_scaling_factor.
 *   topk_ids     int32 [T,k]  experts in selection order (best first).
 *   topk_weights fp32  [T,k]  same order.
 * Checks: 1 <= T, 1 <= E <= MOE_MAX_EXPERTS, 1 <= k <= min(E, MOE_MAX_TOPK);
 * grouped mode: n_group divides E, 1 <= topk_group <= n_group <= 32,
 * k <= topk_group * E / n_group. */
moe_status_t moe_router_topk(const float* logits, const float* correction_bias, int T, int E,
                             int top_k, int mode, int n_group, int topk_group, int renormalize,
                             float routed_scaling_factor, int32_t* topk_ids, float* topk_weights,
                             moe_stream_t stream);

/* moe_router_gemm_topk: the router linear and the top-k in one call:
 *     logits = x . W_r (+ logit_bias), then moe_router_topk's selection.
 * The pages give no arithmetic for the router linear ([65207] "Purpose" passes
 * the gate linear's output to the top-k); this call defines one fixed fp32
 * order so that its logits, and every decision taken from them, can be
 * reproduced bit for bit on any machine:
 *     c = H / 8; p_j = fp32 running sum of x[t,h] * W_r[h,e] over
 *     h = j*c .. j*c + c - 1 in index order (j = 0..7);
 *     logit = (...((p_0 + p_1) + p_2) + ...) + p_7, then + logit_bias[e].
 * Every addition rounds to nearest fp32; products of bf16 or fp16 values are
 * exact in fp32, so they do not round (products below the fp32 normal range,
 * impossible for fp16 and absent for bf16 inputs of ordinary magnitude, would).
 * One cluster of 8 CTAs per 4 tokens (16 once T >= 64 and E <= 256): CTA j
 * sums chunk j, streaming its rows of W_r through shared memory by bulk copy,
 * and writes its partial sums into CTA 0's shared memory (distributed shared
 * memory); CTA 0 adds them in chunk order and selects.
 *   dtype       MOE_DT_BF16 or MOE_DT_FP16: the type of x and W_r.
 *   x           [T,H] row-major; W_r [H,E] row-major (E contiguous).
 *   logit_bias  fp32 [E] or NULL, added to the logits before routing.
 *   logits      fp32 [T,E] output or NULL: the logits the routing used.
 *   other arguments, outputs and checks: as moe_router_topk, plus
 *   H % 8 == 0 and E % 8 == 0 (MOE_ERR_SHAPE), W_r 16-byte aligned
 *   (MOE_ERR_ALIGNMENT); MOE_ERR_SHAPE also if the shared-memory layout does
 *   not fit one CTA (H = 7168 with E = 512 fits). */
moe_status_t moe_router_gemm_topk(int dtype, const void* x, const void* w_r, const float* logit_bias,
                                  const float* correction_bias, int T, int H, int E, int top_k,
                                  int mode, int n_group, int topk_group, int renormalize,
                                  float routed_scaling_factor, float* logits, int32_t* topk_ids,
                                  float* topk_weights, moe_stream_t stream);

/* moe_align_sort: group the T*k routed slots by expert for the grouped GEMMs
 * ([65207] reviewer measurements: moe_sorting; here it never zeroes the layer
 * output - the stage-2 epilogue owns the output; [6106]: the GEMM rows follow
 * this gather index).
 *   topk_ids      int32 [T,k]; slot f = t*k + j.
 *   sorted_ids    int32 [>= moe_sorted_capacity]: experts in order 0..E-1;
 *                 inside an expert ascending f (stable); every expert segment
 *                 padded to a multiple of block_m with the sentinel T*k.
 *                 Entries at and past *num_padded are not written.
 *   block_expert  int32 [>= capacity/block_m]: owning expert of each block.
 *   expert_counts int32 [E]; expert_offsets int32 [E+1] (padded prefix sum);
 *   num_padded    int32 [1] = expert_offsets[E].
 * Checks: block_m in {16,32,64,128,256}; T*k <= 1<<20; E <= MOE_MAX_EXPERTS.
 * An expert id outside [0,E) sets device error 2 and is dropped.
 * One CTA of 1024 threads below 4096 slots; from 4096 on, a cluster of 8 such
 * CTAs, each sorting its eighth of the slots and reading the others' per-expert
 * counts over distributed shared memory (the results are the same). */
moe_status_t moe_align_sort(const int32_t* topk_ids, int T, int top_k, int E, int block_m,
                            int32_t* sorted_ids, int32_t* block_expert, int32_t* expert_counts,
                            int32_t* expert_offsets, int32_t* num_padded, moe_stream_t stream);

/* moe_append_shared_slots: the shared expert as always-selected routed
 * experts ([61503] "Fused heterogeneous MoE", "Overview"). When the caller
 * has appended the shared expert to the routed weights as m virtual experts
 * E..E+m-1 (I intermediate features each, the last zero-padded past Is), this
 * call extends every token's top-k by those m slots:
 *   out_ids[t, 0..k-1] = topk_ids[t, :], out_ids[t, k+v] = E + v;
 *   out_weights likewise, the appended slots weighted by gate[t] (bf16 or
 *   fp16 per gate_dtype) or 1 when gate is NULL.
 * moe_align_sort (E + m experts, k + m slots) and the two grouped GEMMs then
 * compute routed and shared experts in the same launches, and stage 2 sums
 * all k + m contributions before its one rounding (no addend, no side
 * stream). Checks: E + m <= MOE_MAX_EXPERTS, k + m <= MOE_MAX_TOPK. */
moe_status_t moe_append_shared_slots(const int32_t* topk_ids, const float* topk_weights, int T, int top_k,
                                     int E, int m, const void* gate, int gate_dtype, int32_t* out_ids,
                                     float* out_weights, moe_stream_t stream);

/* moe_quantize_activations: the layer's bf16 activations x [T,H] to the
 * stage-1 operand formats, so that bf16 x can enter an fp8 or MXFP8 layer
 * ([6106] "Technical Details": per-token activation scales; BLOCK_K = 32).
 *   dtype MOE_DT_FP8_E4M3: scale fp32 [T], s = amax(x_t)/448 (1 for an
 *         all-zero row); codes [T,H] = e4m3(x / s), the quotient an IEEE fp32
 *         division, round to nearest even, saturating to +-448.
 *   dtype MOE_DT_MXFP8_E4M3: scale = ue8m0 bytes [T, H/32], X + 127 with
 *         X = floor(log2 amax) - 8 per 32 columns (clamped to [-127,127],
 *         -127 for an all-zero block); codes e4m3(x * 2^-X).
 * One CTA per token row. Checks: H % 8 == 0 (fp8) / % 32 == 0 (MXFP8),
 * H <= 16384, x 16-byte aligned, codes 8-byte aligned. Asynchronous on
 * `stream`. */
moe_status_t moe_quantize_activations(int dtype, const void* x, int T, int H, void* codes, void* scale,
                                      moe_stream_t stream);

/* moe_stage1_gemm: per sorted row r (slot f = sorted_ids[r], token t = f/k,
 * expert e = block_expert[r/block_m]):
 *     a   = W13[e] . x[t]                           (2I outputs, fp32 accumulate)
 *     a  *= x_scale[t] * w13_scale[e]               (MOE_DT_FP8_E4M3; [6106])
 *     h_r = SiLU(a[0:I]) * a[I:2I]
 * then h_r is stored in the stage-2 operand format ([6106]: quantisation fused
 * after the activation). tcgen05 tensor cores, weights streamed by TMA; token
 * rows (and MXFP8 token scales) copied into sorted order by a preparation
 * kernel launched first on `stream`, then read one box per 128-byte K atom. The
 * preparation kernel records device error 3 for a sorted slot id that is
 * neither a slot nor the padding value T*top_k.
 *   dtype      MOE_DT_BF16, MOE_DT_FP8_E4M3, MOE_DT_MXFP8_E4M3 or
 *              MOE_DT_MXFP4_E2M1 (which reads as MXFP8 below except for W13).
 *   x          [T,H] bf16 or e4m3 codes; x_scale fp32 [T] (FP8), ue8m0 bytes
 *              [T,H/32] row-major (MXFP8), or NULL (BF16).
 *   w13        [E,2I,H]: rows 0..I-1 gate, I..2I-1 up (K = H contiguous);
 *              w13_scale fp32 [E] (FP8), the packed scale tiles of
 *              moe_mx_pack_weight_scales(0, ...) (MXFP8, MXFP4), or NULL.
 *              MXFP4: e2m1 codes, H/2 bytes per row, 32-byte aligned.
 *   sorted_ids / block_expert / num_padded: from moe_align_sort with the same
 *              block_m. sorted_ids == NULL selects identity routing (row r =
 *              token r, expert 0, rows padded to a multiple of block_m; used
 *              for the shared expert, E = 1, k = 1); block_expert and
 *              num_padded are then ignored.
 *   h          [capacity rows, I] (padded rows hold don't-care values):
 *              BF16: bf16. FP8 / MXFP8: e4m3 codes.
 *   h_scale    FP8: fp32 [capacity rows], amax(h_r)/448 (1 for an all-zero
 *              row); the codes are e4m3(h_r / h_scale[r]), round to nearest
 *              even, saturating. MXFP8: moe_mx_h_scale_bytes(...) bytes of
 *              scale tiles, one ue8m0 byte X+127 per (row, 32 columns) with
 *              X = floor(log2 amax) - 8 (clamped to [-127,127], -127 for an
 *              all-zero block) and codes e4m3(h * 2^-X); tile layout as in
 *              moe_mx_pack_weight_scales with the block_m rows of one token
 *              block per tile. NULL for BF16.
 *   ws         moe_stage1_workspace_bytes(...) bytes, zeroed once by the
 *              caller; may be NULL only for BF16 identity routing.
 * Checks: H % 64 == 0 (bf16) / % 128 == 0 (fp8, MXFP8), I % 64 == 0 (% 128
 * for MXFP8), block_m in {16,32,64,128,256} (<= 128 for MXFP8), 16-byte
 * aligned x, w13, h, ws and the MXFP8 scale arrays. */
moe_status_t moe_stage1_gemm(int dtype, const void* x, const void* x_scale, const void* w13,
                             const void* w13_scale, const int32_t* sorted_ids,
                             const int32_t* block_expert, const int32_t* num_padded, int T,
                             int top_k, int H, int I, int E, int block_m, void* h, void* h_scale,
                             void* ws, moe_stream_t stream);

/* moe_stage2_gemm_accumulate: per sorted row r (slot f, token t, expert e):
 *     y_r   = W2[e] . h_r                           (H outputs, fp32 accumulate)
 *     y_r  *= h_scale_r * w2_scale[e]               (MOE_DT_FP8_E4M3; [6106])
 *     out[t] = bf16( addend[t] + sum over the k slots of t of weight[f] * y_r )
 * The top-k weight, the scatter-reduce over the k slots of a token and the
 * shared-expert addend all happen in this GEMM's epilogue ([65207] "Purpose",
 * commit 2): no separate scale, add or zeroing kernel runs. Partial sums meet
 * in an fp32 workspace; the epilogue that brings a token's last slot adds the
 * addend, rounds once to bf16, writes out and re-zeroes its workspace slice.
 *   dtype       as stage 1; h / h_scale are stage 1's outputs.
 *   w2          [E,H,I] (K = I contiguous); w2_scale fp32 [E] (FP8), the
 *               tiles of moe_mx_pack_weight_scales(1, ...) (MXFP8, MXFP4; the
 *               block scales enter the tensor-core MMA), or NULL. MXFP4: e2m1
 *               codes, I/2 bytes per row, 32-byte aligned.
 *   weights     [T*k] per slot f (routing weights, scale folded in), dtype
 *               weights_dtype = MOE_DT_F32, or MOE_DT_BF16 / MOE_DT_FP16 (the
 *               shared gate's output); NULL = 1.0.
 *   addend      bf16 [T,H] or NULL. addend_ready: event recorded after the
 *               addend was written, or NULL; the call makes `stream` wait on it
 *               right before the GEMM ([65207]: only right before stage 2).
 *               addend may equal out (in-place accumulate).
 *   acc_ws      moe_stage2_workspace_bytes(T,H) bytes, zeroed once by the
 *               caller; unused (may be NULL) when top_k == 1.
 *   out         bf16 [T,H]; every token row is written exactly once.
 * Identity routing (sorted_ids == NULL): as in stage 1; with top_k == 1 each
 * row's result goes straight to out (this is how the shared expert's output
 * becomes the addend of the routed call).
 * Checks: H % 128 == 0, I % 64 == 0 (% 128 for MXFP8), block_m as stage 1,
 * 16-byte aligned h, w2, out, addend, acc_ws and the MXFP8 scale arrays. */
moe_status_t moe_stage2_gemm_accumulate(int dtype, const void* h, const void* h_scale,
                                        const void* w2, const void* w2_scale, const void* weights,
                                        int weights_dtype, const int32_t* sorted_ids,
                                        const int32_t* block_expert, const int32_t* num_padded,
                                        int T, int top_k, int H, int I, int E, int block_m,
                                        const void* addend, moe_event_t addend_ready, void* acc_ws,
                                        void* out, moe_stream_t stream);

/* Size of the stage-2 workspace that the library itself holds in device memory
 * for moe_stage2_gemm_accumulate_static_ws (8 MiB on every GPU that loads the
 * library, kept until the process exits). */
#define MOE_STAGE2_STATIC_WS_BYTES (8u << 20)

/* moe_stage2_gemm_accumulate_static_ws: moe_stage2_gemm_accumulate for callers
 * that cannot allocate device memory themselves - plugin interfaces that hand
 * the operator only its input and output buffers, or processes whose device
 * memory has already been handed to another allocator's pool, where a
 * cudaMalloc would fail or could synchronise the device. There is no
 * counterpart of this call in the pages; it exists for those callers.
 *
 * Arguments and results are those of moe_stage2_gemm_accumulate without
 * acc_ws. In its place the library uses a statically allocated device array of
 * MOE_STAGE2_STATIC_WS_BYTES. This call allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *   - Limit: top_k > 1 needs moe_stage2_workspace_bytes(T, H) <=
 *     MOE_STAGE2_STATIC_WS_BYTES (for H = 2048 up to T = 1016); larger
 *     problems return MOE_ERR_WORKSPACE_LIMIT (message in
 *     moe_last_cuda_error()) and launch nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture. The address is kept for the life of the
 *     process: after a cudaDeviceReset it is stale, so do not call this entry
 *     point again in a process that has reset the device.
 *   - `stream` must belong to the current device (MOE_ERR_DEVICE otherwise:
 *     the array used is the current device's).
 *   - The array is shared by every call on a device and keeps the last call's
 *     contents; each call clears the part it uses on `stream` before its
 *     kernel. Calls whose work overlaps on the GPU (concurrent streams) race
 *     on the array: serialise them. */
moe_status_t moe_stage2_gemm_accumulate_static_ws(int dtype, const void* h, const void* h_scale,
                                                  const void* w2, const void* w2_scale,
                                                  const void* weights, int weights_dtype,
                                                  const int32_t* sorted_ids,
                                                  const int32_t* block_expert,
                                                  const int32_t* num_padded, int T, int top_k,
                                                  int H, int I, int E, int block_m,
                                                  const void* addend, moe_event_t addend_ready,
                                                  void* out, moe_stream_t stream);

/* shared_expert_gate_dot: out[t] = sigmoid(sum_k x[t,k] * w[k]) ([56789]),
 * one fused kernel, fp32 accumulation, the result stored in x's dtype (the
 * store rounds). apply_sigmoid == 0 stores the plain dot.
 *   dtype MOE_DT_BF16 or MOE_DT_FP16 (x, w and out share it).
 *   x [T,K], w [K], out [T]. Checks: T >= 1, K >= 1. */
moe_status_t shared_expert_gate_dot(int dtype, const void* x, const void* w, int T, int K,
                                    int apply_sigmoid, void* out, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
