/*
 * moe.h - C ABI of libmoe_b200.so, a fused Mixture-of-Experts layer for one
 * NVIDIA B200 (sm_100a).
 *
 * The calls follow the problem statement of "Mixture-of-Experts kernel
 * engineering on Amazon SageMaker AI" (abstract, the "fused MoE" passage): a
 * fused MoE layer is token routing, data shuffling, the experts' network math
 * and expert aggregation, run as one batched GPU operation instead of a loop
 * of separate steps.  Each step has its own entry point here, and
 * moe_fused_forward runs them all back to back on one stream.
 *
 * Conventions shared by every call
 *   - All pointers except the moe_shape_t are DEVICE pointers that the caller
 *     allocated; the library allocates nothing in these calls and keeps no
 *     pointer after a call returns.  Calls are asynchronous on `stream`
 *     (a cudaStream_t; NULL = the legacy default stream), never synchronise
 *     the device and never copy device data to the host, so a sequence of
 *     calls can be captured into a CUDA graph.
 *   - Return value: MOE_OK, or a negative moe_status code for argument errors
 *     found on the host before anything is launched.  Errors found by the
 *     kernels (an expert id out of range, a mis-aligned segment, a pipeline
 *     wait that timed out) are written to a status word inside the workspace;
 *     read it with moe_get_device_status after the stream has completed.
 *   - bf16 tensors are IEEE bfloat16, FP8 tensors are E4M3 ("fn": bias 7, no
 *     infinities, largest finite 448); real value = code * scale.
 *   - Row-major, K-major storage: element (r, c) of an [R, C] matrix lives at
 *     r*C + c.  Expert weights are stacked along a leading expert axis.
 *   - Shared (always-on) experts are stored after the E routed experts in
 *     every per-expert array (weights and scales), i.e. shared expert s has
 *     expert index E + s.
 *   - Rows: the routed rows of the layer are the flat indices f = t*k + j of
 *     (token t, choice j); shared expert s adds the row codes T*k + s*T + t.
 *     Each expert's rows form one contiguous segment of a row-permuted
 *     buffer, segments in expert order, each padded to a multiple of `pad`
 *     rows.  Every such buffer is sized for moe_max_rows() rows, an upper
 *     bound the host computes without reading routing results.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* = cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,        /* null pointer, bad size, k > E, ...      */
    MOE_ERR_UNSUPPORTED = -2,        /* valid, but a shape/dtype not built      */
    MOE_ERR_WORKSPACE_TOO_SMALL = -3,
    MOE_ERR_CUDA = -4,               /* a CUDA runtime/driver call failed       */
    MOE_ERR_DEVICE_CHECK = -5,       /* a kernel found bad data (device status) */
    MOE_ERR_TIMEOUT = -6             /* a kernel wait gave up (device status)   */
} moe_status;

enum { MOE_BF16 = 0, MOE_E4M3 = 1 };
enum { MOE_GATE_SOFTMAX = 0, MOE_GATE_SIGMOID = 1 };
enum { MOE_VARIANT_AUTO = 0, MOE_VARIANT_SWAP_AB = 1, MOE_VARIANT_NORMAL = 2 };

/*
 * Problem description, passed by pointer to every call (host memory, read
 * during the call only).
 *   T        tokens in this call (>= 1).  A runtime value: no call is ever
 *            specialised or recompiled for a token count (the lesson of the
 *            Russian summary's section "Убрать лишние JIT-перекомпиляции
 *            Triton": a recompile per num_tokens costs time-to-first-token).
 *   H, I     hidden size and expert intermediate size; multiples of 128.
 *   E, k     routed experts (1..512) and experts chosen per token (1..min(E,32)).
 *   n_shared always-on shared experts (0 or 1), same I as the routed ones.
 *   gate     MOE_GATE_SOFTMAX: w = softmax of the chosen logits (renorm) or
 *            the full softmax entry (no renorm).  MOE_GATE_SIGMOID:
 *            s = sigmoid(logit); w = s / sum of chosen s (renorm) or s.
 *   renorm   see gate.
 *   routed_scale  multiplies every routed weight (1.0 for Mixtral, 2.5 for a
 *            DeepSeek-V3-shaped layer).  Shared experts have weight 1.
 *   wdtype   weight dtype (MOE_BF16, or MOE_E4M3 with one fp32 scale per
 *            expert matrix).
 *   adtype   dtype the expert GEMMs read activations in: MOE_BF16, or MOE_E4M3
 *            (tokens quantised with the static scale a1 by the gather step,
 *            the hidden vector with the static scale a2 by the first GEMM).
 *            MOE_E4M3 requires wdtype == MOE_E4M3.
 *   pad      segment padding in rows: a multiple of 16 (16..256) for the GEMM
 *            calls; any value >= 1 for moe_align_permute alone.
 *   variant  GEMM operand order: MOE_VARIANT_SWAP_AB puts the expert weight
 *            rows in the tensor core's M slot and the tokens in N (the
 *            "Swap-AB" of the AWS post, B^T[N,K] x A^T[K,M] = C^T[N,M], used
 *            when an expert sees few rows); MOE_VARIANT_NORMAL puts token rows
 *            in M; MOE_VARIANT_AUTO picks Swap-AB when no expert can receive more
 *            than 128 rows (T <= 128; 128 is the fixed M extent of a one-SM
 *            tcgen05.mma), else normal.  Results are the same up to fp32
 *            summation order.  E4M3 weights with bf16 activations always
 *            use Swap-AB.
 */
typedef struct {
    int32_t T, H, I, E, k, n_shared;
    int32_t gate, renorm;
    float routed_scale;
    int32_t wdtype, adtype;
    int32_t pad;
    int32_t variant;
} moe_shape_t;

/* Rows every row-permuted buffer (sorted_rows, xp, h, y) must hold:
 * T*k + n_shared*T + (E + n_shared)*(pad - 1). */
int moe_max_rows(const moe_shape_t *shape, int64_t *rows);

/* Bytes of workspace moe_fused_forward needs (the other calls need no more).
 * The workspace must be 256-byte aligned; its contents need no initialisation
 * and are overwritten by every call. */
int moe_workspace_size(const moe_shape_t *shape, size_t *bytes);

/*
 * Step 1 - token routing (top-k gating over router logits).
 *   logits [T, E] fp32 in; ids [T, k] int32 and w [T, k] fp32 out.
 *   Per token the k experts of largest logit, in descending order; equal
 *   logits go to the lower expert id; NaN ranks below every number.  Weights
 *   as described for moe_shape_t.gate, times routed_scale.  Selection is on
 *   the logit, so it is exact and reproducible.
 */
int moe_route_topk(const moe_shape_t *shape, const float *logits, int32_t *ids, float *w,
                   moe_stream_t stream);

/*
 * Step 0+1 - router logits and top-k in one launch (the Chinese retelling,
 * section "2. 用于FP8量化的Triton后端路由": routing is decided inside the
 * fused kernel, without host control flow).
 *   x [T, H] bf16 and wg [E, H] bf16 (the router weight) in, both 16-byte
 *   aligned; logits [T, E] fp32, ids [T, k] and w [T, k] out, ids and w as
 *   for moe_route_topk on those logits.
 *   logits[t,e] = sum_h x[t,h] * wg[e,h] in a fixed order, so that routing is
 *   reproducible bit for bit: in double precision, 32 partial sums where sum
 *   l takes, in ascending h, the 8-element chunks h/8 congruent to l mod 32;
 *   then s_l += s_(l xor o) for o = 16, 8, 4, 2, 1; one rounding to fp32.
 *   ws: workspace of moe_workspace_size bytes (per-token tickets).
 * Errors: MOE_ERR_INVALID_ARG for NULL or misaligned pointers,
 * MOE_ERR_WORKSPACE_TOO_SMALL.
 */
int moe_router_topk(const moe_shape_t *shape, const void *x, const void *wg, float *logits, int32_t *ids,
                    float *w, void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Step 2 - alignment / permutation ("data shuffling").
 *   ids [T, k] int32 in (each in 0..E-1).  Out:
 *     counts      [E + n_shared]   rows of each expert (T for shared experts)
 *     offsets     [E + n_shared+1] first slot of each segment; last = total
 *     sorted_rows [max_rows]       slot -> row code, -1 for pad slots; slots at
 *                                  or beyond offsets[E + n_shared] untouched
 *     inv         [T*k]            routed row f -> its slot
 *   Within a segment rows are in ascending row code (a stable counting sort):
 *   the result is deterministic and bit-exact.  An id outside 0..E-1 sets
 *   MOE_ERR_DEVICE_CHECK in the device status and that row is dropped.
 *   ws: workspace of moe_workspace_size bytes (histogram scratch + status).
 */
int moe_align_permute(const moe_shape_t *shape, const int32_t *ids, int32_t *counts,
                      int32_t *offsets, int32_t *sorted_rows, int32_t *inv, void *ws,
                      size_t ws_bytes, moe_stream_t stream);

/*
 * Step 2 without a workspace (no counterpart on the pages: an addition for
 * callers that cannot allocate).  Some callers cannot provide the `ws` buffer
 * the call above needs -- for example an engine whose device memory is all
 * reserved by its own allocator at start-up, or a latency-critical loop that
 * may not call cudaMalloc because it can synchronise the device.  This call
 * computes exactly what moe_align_permute computes, but keeps its scratch
 * (per-block histograms and control words, 262,912 bytes) in one fixed array
 * inside the library, held on every GPU that loads the library until the
 * process exits.  It allocates nothing.
 *   Limits: T*k <= 65536 routed rows and E + n_shared <= 513 experts; larger
 *   shapes return MOE_ERR_UNSUPPORTED before anything is launched.
 *   status: optional device int32 (may be NULL) that receives the call's
 *   device status (MOE_ERR_DEVICE_CHECK for an id outside 0..E-1).
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) while that device is current; make that first call
 *   before any stream capture.  The address is kept for the life of the
 *   process: after cudaDeviceReset on a device, do not call this entry point
 *   on that device again.  Devices with an index of 64 or more return
 *   MOE_ERR_UNSUPPORTED.  All calls share the one array, so calls that
 *   overlap on the GPU (different streams, or different host threads using
 *   the same device) race and must be serialised by the caller.  The status
 *   word inside the array is cleared at the start of every call, so an error
 *   reported by one call does not carry over to the next.
 */
int moe_align_permute_noalloc(const moe_shape_t *shape, const int32_t *ids, int32_t *counts,
                              int32_t *offsets, int32_t *sorted_rows, int32_t *inv,
                              int32_t *status, moe_stream_t stream);

/*
 * Step 3 - gather the tokens into expert order.
 *   x [T, H] bf16 in; xp [max_rows, H] out, slot s = x[token of sorted_rows[s]]
 *   (zeros for pad slots).  adtype == MOE_E4M3: xp holds E4M3 codes of
 *   fp32(x) / a1_scale (IEEE fp32 quotient, round-to-nearest-even, saturated
 *   to +-448); otherwise bf16, copied bit for bit.
 */
int moe_gather(const moe_shape_t *shape, const void *x, const int32_t *sorted_rows,
               const int32_t *offsets, float a1_scale, void *xp, moe_stream_t stream);

/*
 * Step 4 - grouped expert GEMM for the gate and up projections with the
 * SwiGLU epilogue.  For each slot s of expert e's segment:
 *     g = (xp_s . W1[e]^T) * sc,  u = (xp_s . W3[e]^T) * sc,
 *     h_s = SiLU(g) * u,          sc = a1_scale * w13_scale[e]
 * (a1_scale = 1 for bf16 activations; w13_scale NULL means all ones).
 *   xp  [max_rows, H] (adtype), w13 [E + n_shared, 2I, H] (wdtype; rows 0..I-1
 *   of each expert are W1 = gate, rows I..2I-1 are W3 = up), offsets as from
 *   step 2.  h [max_rows, I] out: bf16, or for adtype == MOE_E4M3 the E4M3
 *   codes of h / a2_scale (saturated).  Only rows of segments are written.
 *   fp32 accumulation in tensor memory.  In the Swap-AB variant an expert's
 *   weight tile is streamed once per row tile of its segment: once when the
 *   segment fits one tile (256 rows, or 16 rows for E4M3 weights with bf16
 *   activations); the row tiles of one weight tile run side by side, so a
 *   repeat read comes mostly from L2.
 *   E4M3 weights with bf16 activations (this call and step 5): the
 *   activation rows are first split, in the workspace, into two E4M3 planes
 *   with one power-of-two scale s per row, v = s * (hi + lo), and the GEMM
 *   runs on the E4M3 tensor path.  The split is exact except for elements
 *   below about 2^-11 of their row's largest magnitude, which are off by at
 *   most 2^-10 s.
 */
int moe_grouped_gemm_swiglu(const moe_shape_t *shape, const void *xp, const void *w13,
                            const float *w13_scale, float a1_scale, float a2_scale,
                            const int32_t *offsets, void *h, void *ws, size_t ws_bytes,
                            moe_stream_t stream);

/*
 * Step 5 - grouped down-projection GEMM: y_s = (h_s . W2[e]^T) * a2_scale *
 * w2_scale[e] for each slot s of expert e.
 *   h [max_rows, I] (adtype), w2 [E + n_shared, H, I] (wdtype), y [max_rows, H]
 *   fp32 out (rows of segments only).
 */
int moe_grouped_gemm_down(const moe_shape_t *shape, const void *h, const void *w2,
                          const float *w2_scale, float a2_scale, const int32_t *offsets,
                          float *y, void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Step 6 - weighted combine back to token order ("expert aggregation"):
 *   out[t] = sum_{j<k} w[t,j] * y[inv[t*k+j]] + sum_s y[offsets[E+s] + t]
 * summed in fp32 in that fixed order, written as bf16 (round to nearest even).
 *   y [max_rows, H] fp32, w [T, k] fp32, inv [T*k], offsets [E+n_shared+1];
 *   out [T, H] bf16.
 */
int moe_combine(const moe_shape_t *shape, const float *y, const float *w, const int32_t *inv,
                const int32_t *offsets, void *out, moe_stream_t stream);

/*
 * The whole layer in one call: steps 1-6 on `stream` with every
 * intermediate in the workspace.  x [T, H] bf16, logits [T, E] fp32,
 * w13/w2 and scales as above (scales may be NULL for bf16 weights),
 * a1_scale/a2_scale the static activation scales (ignored for bf16
 * activations), out [T, H] bf16.
 */
int moe_fused_forward(const moe_shape_t *shape, const void *x, const float *logits,
                      const void *w13, const float *w13_scale, const void *w2,
                      const float *w2_scale, float a1_scale, float a2_scale, void *out,
                      void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The same layer starting from the router weight: step 0+1
 * (moe_router_topk, logits kept in the workspace) instead of step 1.
 * wg [E, H] bf16, 16-byte aligned; everything else as moe_fused_forward.
 */
int moe_fused_forward_router(const moe_shape_t *shape, const void *x, const void *wg, const void *w13,
                             const float *w13_scale, const void *w2, const float *w2_scale,
                             float a1_scale, float a2_scale, void *out, void *ws, size_t ws_bytes,
                             moe_stream_t stream);

/*
 * Attention-side step: inverse rotary embedding fused with per-head E4M3
 * quantisation ("_fused_inv_rope_fp8_quant_per_head" in the Russian summary,
 * section "Убрать лишние JIT-перекомпиляции Triton": rotary embedding and FP8
 * quantisation in one kernel, whose recompilation for every new num_tokens
 * cost 9% of time-to-first-token until the token count was made a run-time
 * value).  num_tokens is a run-time value here; nothing is built per count.
 *   num_tokens  tokens (>= 0; 0 is a no-op)
 *   n_heads     heads per token (>= 1)
 *   head_dim    64, 128 or 256
 *   rot_dim     rotated elements per head, at most head_dim: even for
 *               interleaved pairs, a multiple of 16 for neox pairs
 *               (MOE_ERR_UNSUPPORTED otherwise); the rest pass through
 *               unrotated
 *   max_pos     rows of the rotary table
 *   interleaved 0: pairs (i, i + rot_dim/2) ("neox"); 1: pairs (2i, 2i+1)
 */
typedef struct {
    int32_t num_tokens, n_heads, head_dim, rot_dim, max_pos, interleaved;
} moe_rope_shape_t;

/*
 *   x [num_tokens, n_heads, head_dim] bf16 (16-byte aligned), positions
 *   [num_tokens] int32, cos_sin [max_pos, rot_dim] fp32 (row p: cos(p w_i)
 *   for i < rot_dim/2, then sin(p w_i)) in; q [num_tokens, n_heads, head_dim]
 *   E4M3 codes (8-byte aligned) and scales [num_tokens, n_heads] fp32 out.
 *   Each pair (a', b') of a head is rotated back by its token's angle,
 *   a = a' c + b' s, b = b' c - a' s; then scale = amax(|r|)/448 per (token,
 *   head) (1 if all zero) and q = E4M3(r / scale), round to nearest even,
 *   saturated.  fp32 arithmetic, each product and sum rounded on its own, IEEE
 *   division: the codes are reproducible bit for bit.
 *   status: optional device int32 (may be NULL); a position outside
 *   [0, max_pos) sets it to MOE_ERR_DEVICE_CHECK (if it was 0) and gives that
 *   token zero codes and scale 0.  Otherwise it is left unchanged.
 * Errors: MOE_ERR_INVALID_ARG (bad sizes, NULL or misaligned pointers),
 * MOE_ERR_UNSUPPORTED (other head_dim).  Asynchronous on `stream`.
 */
int moe_inv_rope_quant_per_head(const moe_rope_shape_t *shape, const void *x, const int32_t *positions,
                                const float *cos_sin, uint8_t *q, float *scales, int32_t *status,
                                moe_stream_t stream);

/*
 * Self-test of the failure path (no counterpart on the pages): launches one
 * block whose two bounded pipeline waits run out, because nothing arrives on
 * their barriers.  The first gives up after the library's wait limit (2 s),
 * raises the block's abort flag, and the second then gives up at once.  The
 * block writes MOE_ERR_TIMEOUT to the status word at the start of `ws` and
 * exits, so the CUDA context stays usable.  gave_up (device int32) receives
 * the number of waits that gave up (2).  Asynchronous on `stream`.
 */
int moe_selftest_wait_timeout(void *ws, int32_t *gave_up, moe_stream_t stream);

/*
 * Self-test of the CTA-pair abort path (no counterpart on the pages): the
 * down projection of moe_grouped_gemm_down (same arguments; bf16 weights and
 * activations, a shape on the normal order: more than 128 tokens, or
 * variant MOE_VARIANT_NORMAL), except that in every CTA pair the second CTA
 * stops loading its half of the operands after two stages.  The first CTA's
 * waits for those stages run out after the wait limit (2 s); both CTAs then
 * take the pair's abort tear-down (no copy left in flight into either CTA,
 * tensor memory freed), MOE_ERR_TIMEOUT goes to the status word at the start
 * of `ws`, and the kernel exits, so the CUDA context stays usable.  The
 * experts handled by one-CTA tiles are computed normally; y of the experts
 * on pairs is undefined.  Returns MOE_ERR_UNSUPPORTED for other shapes.
 * Asynchronous on `stream`.
 */
int moe_selftest_pair_abort(const moe_shape_t *shape, const void *h, const void *w2, const int32_t *offsets,
                            float *y, void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Device status written by the kernels into `ws`: copies it to *status
 * (host) after synchronising `stream` -- the one call here that waits.
 * MOE_OK when no kernel reported a problem since the last reset.
 */
int moe_get_device_status(const void *ws, int32_t *status, moe_stream_t stream);

/* Zero the device status word (asynchronous on `stream`). */
int moe_reset_device_status(void *ws, moe_stream_t stream);

/* Human-readable text for a moe_status value (static storage). */
const char *moe_status_string(int status);

/* Number of this library's kernel launches the last call on this host thread
 * issued (for launch accounting). */
int moe_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
