/*
 * moe_dispatch_combine.h -- C ABI of the B200 MoE token dispatch / combine library.
 *
 * What the calls compute
 * ----------------------
 * "Enabling trillion-parameter models on AWS EFA", section "Introdução" and
 * section "MoE all-to-all sobre EFA": a dispatch step takes the tokens and the
 * experts chosen for each token and sends each token to where its experts live;
 * its dual, combine, takes the experts' processed rows back and forms each
 * token's routing-weighted sum.  Section "Buffers de Envio e Recebimento" and
 * section "Despacho e Combinação" of the same page fix the layout: tokens are
 * counted per expert, the cumulative sum of the counts gives each expert's
 * offset, and each expert's tokens are packed contiguously from there.  Section
 * "Avaliação" evaluates the dispatch with block-scaled fp8 payloads and the
 * combine in bf16; "Lower latency and higher throughput with multi-node
 * DeepSeek deployment", section "Quantização", defines the blocks: one scale
 * per 128-element activation vector.
 *
 * On one GPU the "ranks" that host experts are virtual: rank r owns experts
 * [r*E/R, (r+1)*E/R) (the expert-parallel split of the DeepSeek page, section
 * "Paralelismo de Especialistas"), and its receive buffer is the contiguous row
 * range [rank_offset[r], rank_offset[r+1]) of one allocation.
 *
 * Conventions
 * -----------
 * - Every pointer argument except `cfg`, `out`, `handle`, `bits_out` and
 *   `sizes` is a DEVICE pointer.  The caller allocates and owns every buffer;
 *   the library allocates nothing and frees nothing.
 * - All arrays are dense and row-major.  bf16 data is passed as 16-bit IEEE
 *   bfloat16 bit patterns; fp8 data as OCP e4m3 ("e4m3fn") bytes.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call
 *   only enqueues work on it and returns; nothing waits for the GPU except
 *   moe_check.  No call reads data back to the host, so a dispatch/combine
 *   sequence can be captured in a CUDA graph.
 * - Host-side argument errors return a negative status and enqueue nothing.
 * - Device-side errors (an expert id outside [0,E), a receive row at or past
 *   the capacity) never trap: the offending entry is dropped (its slot is -1
 *   and nothing is stored for it) and a bit is OR-ed into the caller's device
 *   error word.  moe_check reads and clears that word.
 */
#ifndef MOE_DISPATCH_COMBINE_H
#define MOE_DISPATCH_COMBINE_H

#include <stddef.h>
#include <stdint.h>

/* Entry points are exported from the shared library; everything else is hidden. */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* moe_config.flags */
#define MOE_FP8 1    /* payload as e4m3 codes plus one fp32 scale per 128 columns */
#define MOE_PAD128 2 /* every expert segment padded to a multiple of 128 rows      */
/* The caller states that x, topk_idx and topk_w were complete before the
 * previous kernel in the stream began (that kernel does not write them): the
 * dispatch may read and compute before waiting for it, and only its writes
 * wait.  moe_dispatch uses it at decode sizes; other calls ignore it, and
 * moe_route_dispatch ignores it (its ids come from its own router). */
#define MOE_INPUTS_READY 4

/* Host status codes. */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG -1 /* a null or misaligned pointer, a bad size        */
#define MOE_ERR_UNSUPPORTED -2 /* a valid request outside what the kernels cover */
#define MOE_ERR_CUDA -3        /* a CUDA runtime call or launch failed            */
#define MOE_ERR_DEVICE -4      /* moe_check: the device error word was non-zero  */
#define MOE_ERR_TOO_LARGE -5   /* moe_dispatch_no_alloc: scratch would not fit    */

/* Bits of the device error word. */
#define MOE_DEV_BAD_INDEX 1 /* dispatch: an expert id outside [0, E)                  */
#define MOE_DEV_CAPACITY 2  /* dispatch: a receive row at or past rows_cap            */
#define MOE_DEV_TIMEOUT 4   /* a bounded device wait gave up                           */
#define MOE_DEV_BAD_SLOT 8  /* payload / combine: a slot outside [-1, rows_cap)        */

/* Router score functions (moe_router_topk). */
#define MOE_SCORE_SOFTMAX 0
#define MOE_SCORE_SIGMOID 1

/* Limits of this library. */
#define MOE_MAX_EXPERTS 2048 /* E */
#define MOE_MAX_TOPK 64      /* k */
#define MOE_NO_ALLOC_SCRATCH_BYTES (1u << 20) /* fixed scratch of moe_dispatch_no_alloc */
#define MOE_EP_MAX_WAIT_NS 10000000000ull   /* longest moe_ep_wait limit: 10 s      */

/*
 * Problem description.
 *   H      hidden size; a multiple of 8 (16-byte rows), and of 128 with MOE_FP8.
 *   k      experts per token, 1..MOE_MAX_TOPK.
 *   E      experts, 1..MOE_MAX_EXPERTS.
 *   R      virtual ranks; E must be a multiple of R.
 *   flags  OR of MOE_FP8, MOE_PAD128.
 */
typedef struct {
    int32_t H, k, E, R, flags;
} moe_config;

/*
 * Caller-allocated dispatch outputs (device pointers).
 *   recv_x        [rows_cap, H] bf16, or [rows_cap, H] e4m3 bytes with MOE_FP8.
 *                 Row slot[t,j] holds token t's payload; 16-byte aligned.
 *   recv_scale    [rows_cap, H/128] fp32 with MOE_FP8 (16-byte aligned), else NULL.
 *   expert_count  [E]     tokens routed to each expert.
 *   expert_offset [E+1]   first row of each expert's segment; expert_offset[E]
 *                         is the number of rows in use.
 *   rank_offset   [R+1]   rank_offset[r] = expert_offset[r*E/R].
 *   recv_src      [rows_cap] the routing entry t*k+j a row holds, -1 for a row
 *                 that holds none (padding and unused capacity).
 *   rows_cap      rows of recv_x / recv_scale / recv_src.  moe_rows_capacity
 *                 gives the worst case; a smaller capacity is allowed, and
 *                 entries that do not fit are dropped with MOE_DEV_CAPACITY.
 * Rows without an entry are not written in recv_x and recv_scale.
 */
typedef struct {
    void *recv_x;
    float *recv_scale;
    int32_t *expert_count;
    int32_t *expert_offset;
    int32_t *rank_offset;
    int32_t *recv_src;
    int64_t rows_cap;
} moe_dispatch_out;

/*
 * What combine needs from a dispatch ("Buffers de Envio e Recebimento": the
 * combine already has the routing information from the dispatch phase).
 * Filled by moe_dispatch; plain data, copyable, valid while the buffers it
 * points to live.
 *   slot    [T, k] int32 device: receive row of entry (t, j), or -1 if dropped.
 *   topk_w  [T, k] fp32 device: the routing weights passed to moe_dispatch.
 */
typedef struct {
    moe_config cfg;
    int32_t T;
    int32_t *slot;
    const float *topk_w;
    int64_t rows_cap;
} moe_handle;

/* Byte sizes of the dispatch buffers for a given capacity (host-only helper). */
typedef struct {
    size_t recv_x, recv_scale, expert_count, expert_offset, rank_offset, recv_src, slot;
} moe_dispatch_sizes;

/*
 * Worst-case receive rows for T tokens: T*k; with MOE_PAD128 the most 128-row
 * blocks T*k entries can fill over min(E, T*k) experts, times 128.
 * Returns -1 for an invalid cfg or T < 0.
 */
MOE_API int64_t moe_rows_capacity(const moe_config *cfg, int32_t T);

/* Fills *sizes for T tokens and rows_cap rows; returns a status. */
MOE_API int moe_dispatch_sizes_for(const moe_config *cfg, int32_t T, int64_t rows_cap,
                           moe_dispatch_sizes *sizes);

/*
 * Bytes of device scratch that moe_dispatch and moe_dispatch_layout require for
 * T tokens (0 for small batches; where moe_dispatch takes a one-launch kernel it
 * leaves the scratch untouched).  Returns 0 and sets nothing for an invalid cfg.
 */
MOE_API size_t moe_workspace_bytes(const moe_config *cfg, int32_t T);

/*
 * Dispatch T tokens (section "Despacho e Combinação" of the EFA page: per-expert
 * counts, their cumulative sum as offsets, tokens packed contiguously per
 * expert).
 *
 *   x         [T, H] bf16, 16-byte aligned.
 *   topk_idx  [T, k] int32 expert ids.
 *   topk_w    [T, k] fp32 routing weights; not read here, only recorded in the
 *             handle for moe_combine (must stay alive until then).
 *   out       caller-allocated outputs, see moe_dispatch_out.
 *   slot      [T, k] int32 output: receive row of each entry, -1 if dropped.
 *   workspace device scratch of at least moe_workspace_bytes(cfg, T) bytes
 *             (may be NULL when that is 0).  Its contents are not preserved.
 *   dev_err   device int32 error word; bits are OR-ed in, never cleared here.
 *   handle    host struct filled on success.
 *
 * Inside each expert's segment, entries are in (token, k) order, so the result
 * is unique and deterministic.  With MOE_FP8 each 128-column block of a token
 * gets scale = amax/448 and codes e4m3(x/scale) (both divisions IEEE binary32
 * round-to-nearest; codes rounded to nearest-even and saturated to +-448; an
 * all-zero block gets scale 0 and codes 0), and every slot of the token gets
 * the same codes and scales.
 * Returns MOE_OK or a negative status (nothing enqueued on error).
 */
MOE_API int moe_dispatch(const moe_config *cfg, int32_t T, const void *x, const int32_t *topk_idx,
                 const float *topk_w, const moe_dispatch_out *out, int32_t *slot,
                 void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream,
                 moe_handle *handle);

/*
 * The two phases of moe_dispatch as separate calls, in the order of the EFA
 * page's section "Despacho e Combinação" (routing information first: counts,
 * their cumulative sum and the offsets that place each token; then the
 * payload is packed).  moe_dispatch_layout followed by moe_dispatch_payload
 * gives exactly the results of moe_dispatch.
 *
 * moe_dispatch_layout: the per-expert counts, offsets, rank offsets, slot[T,k]
 * and recv_src of moe_dispatch; it reads only topk_idx and writes only those
 * arrays of `out` (recv_x / recv_scale may be NULL).  Same workspace rules.
 *
 * moe_dispatch_payload: copies (bf16) or block-quantises (MOE_FP8) each token's
 * row x[t] into rows slot[t, 0..k) of out->recv_x (and out->recv_scale).  The
 * slots normally come from a layout call with the same cfg, T and
 * out->rows_cap.  A slot of -1 is skipped; any other value outside
 * [0, rows_cap) is skipped and sets MOE_DEV_BAD_SLOT, so no write leaves the
 * buffers.  It uses only recv_x, recv_scale and rows_cap of `out`.
 */
MOE_API int moe_dispatch_layout(const moe_config *cfg, int32_t T, const int32_t *topk_idx,
                                const moe_dispatch_out *out, int32_t *slot, void *workspace,
                                size_t workspace_bytes, int32_t *dev_err, void *stream);

MOE_API int moe_dispatch_payload(const moe_config *cfg, int32_t T, const void *x,
                                 const int32_t *slot, const moe_dispatch_out *out,
                                 int32_t *dev_err, void *stream);

/*
 * Combine (EFA page, sections "Introdução" and "Despacho e Combinação"; DeepSeek
 * page, section "Paralelismo de Especialistas"): for every token t,
 *   y[t, :] = bf16( sum_{j=0..k-1} topk_w[t,j] * expert_out[slot[t,j], :] )
 * accumulated in fp32 with one fused multiply-add per j in ascending j,
 * starting from 0, then rounded to nearest-even bf16.  Entries with slot -1
 * are skipped.  The weights are used as given (no division by their sum).
 *
 *   handle      from moe_dispatch.
 *   expert_out  [rows_cap, H] bf16 in the receive layout, 16-byte aligned.
 *   y           [T, H] bf16 output, 16-byte aligned.
 *   dev_err     device error word (may be NULL): MOE_DEV_BAD_SLOT.
 * Returns MOE_OK or a negative status.
 */
MOE_API int moe_combine(const moe_handle *handle, const void *expert_out, void *y, int32_t *dev_err,
                void *stream);

/*
 * Combine with sender-side (per-rank) partial accumulation ("Enabling
 * trillion-parameter models on AWS EFA", section "Avaliação": DeepEP
 * accumulates on the sending side to move less data, which may change
 * precision).  Same inputs as moe_combine plus the dispatch's rank_offset.
 *
 *   1. send: for each token t and each distinct rank r_q among the ranks of
 *      t's kept entries (q in order of first appearance over j; the rank of a
 *      receive row s is the r with rank_offset[r] <= s < rank_offset[r+1]):
 *        partial[t, q, :] = bf16( sum over t's entries j on rank r_q, ascending
 *                                 j, of an fp32 fma of topk_w[t,j] * row )
 *      partial_rank[t, q] = r_q, npart[t] = number of distinct ranks.
 *   2. receive: y[t, :] = bf16( sum_{q < npart[t]} partial[t, q, :] ) in fp32.
 *
 *   rank_offset   [R+1] int32 device (from moe_dispatch).
 *   partial       [T, k, H] bf16 device, 16-byte aligned (the "send buffer";
 *                 rows q >= npart[t] are not written).
 *   partial_rank  [T, k] int32 device;  npart [T] int32 device.
 *   y             [T, H] bf16 device, 16-byte aligned.
 * Compared with moe_combine, each partial is rounded to bf16 once more.
 * Returns MOE_OK or a negative status.
 */
MOE_API int moe_combine_rank_partial(const moe_handle *handle, const int32_t *rank_offset,
                                     const void *expert_out, void *partial,
                                     int32_t *partial_rank, int32_t *npart, void *y,
                                     int32_t *dev_err, void *stream);

/*
 * Expert-side activation: act = e4m3 block quantisation of SiLU(gate) * up
 * ("Lower latency and higher throughput with multi-node DeepSeek deployment",
 * section "Quantização": the SiLU kernel emits block-fp8 activations for the
 * next grouped GEMM and, to stay valid under CUDA graphs with data-dependent
 * routing, runs a fixed set of persistent workers that read how many rows the
 * routing populated).
 *
 *   gate_up      [rows_cap, 2I] bf16 device, 16-byte aligned: gate in columns
 *                [0, I), up in [I, 2I), in a dispatch's receive layout.
 *   recv_src     [rows_cap] int32 device (from moe_dispatch): rows with -1 are
 *                padding and are skipped.
 *   rows_in_use  device int32: rows at or past it are skipped (normally
 *                &expert_offset[E]); clamped to [0, rows_cap].
 *   act          [rows_cap, I] e4m3 bytes device, 16-byte aligned.
 *   act_scale    fp32 device: [rows_cap, I/128] row-major, or with
 *                scale_col_major != 0, [I/128, rows_cap] (one column of scales
 *                per row, the layout grouped GEMMs read).
 * The activation a of a (gate g, up u) pair is the binary32 number nearest to
 * the real value g u / (1 + e^-g) (ties to even; a zero carries the sign of
 * g u); results beyond the binary32 range are out of contract.  Per 128
 * columns: scale = amax/448, codes = e4m3(a/scale) as in moe_dispatch.  I must
 * be a multiple of 128 (else MOE_ERR_UNSUPPORTED).  Rows not selected are left
 * untouched.
 */
MOE_API int moe_silu_quant(int64_t rows_cap, int32_t I, const void *gate_up,
                           const int32_t *recv_src, const int32_t *rows_in_use, void *act,
                           float *act_scale, int32_t scale_col_major, void *stream);

/*
 * The activations of moe_silu_quant alone, for n (gate, up) pairs: act[i] is
 * the binary32 number nearest to g u / (1 + e^-g) for g = gate[i], u = up[i]
 * (bf16 device arrays; "Lower latency and higher throughput with multi-node
 * DeepSeek deployment", section "Quantização": SiLU of the gate times up, the
 * input of the block quantiser).  The kernel takes the same three tiers as
 * moe_silu_quant: for common gates a binary32 product with a table of silu(g)
 * as a pair of binary32 numbers (made at build time) and a certified rounding,
 * else g u sigmoid(g) in fp64 with a certified rounding, and double-double
 * arithmetic near a binary32 rounding boundary; exact_only != 0 takes the
 * double-double tier for every value.  fast_value (fp64 device, may be NULL)
 * receives the fp64 tier's value for each pair (meaningful for finite,
 * nonzero, normal inputs with gate >= -200), for checking its error bound.
 * act is fp32 device.  n = 0 launches nothing.  Returns a status.
 */
MOE_API int moe_silu_mul(int64_t n, const void *gate, const void *up, float *act,
                         double *fast_value, int32_t exact_only, void *stream);

/*
 * Router top-k ("Lower latency and higher throughput with multi-node DeepSeek
 * deployment", section "Roteador MoE": one top-k with index tracking serves all
 * MoE models; plain top-k is group-limited top-k with one group).  For each
 * token's logits[t, 0..E) (fp32 device):
 *   - the experts form n_group contiguous groups of E/n_group; a group's score
 *     is its largest logit; the topk_group best groups are kept (ties: lower
 *     group id);
 *   - the k largest logits among the kept groups' experts are chosen, best
 *     first (ties: lower expert id) -> topk_idx[t, 0..k) (int32 device);
 *   - topk_w[t, j] (fp32 device): MOE_SCORE_SOFTMAX: exp(l_j - m) divided by
 *     the sum over the k chosen (renormalize != 0) or over all E logits;
 *     MOE_SCORE_SIGMOID: 1/(1+exp(-l_j)), divided by the chosen ones' sum when
 *     renormalize != 0.
 * The choice compares logits only (both score functions are increasing), so
 * it is exact.  Limits: E <= 1024, k <= 32, n_group <= 32, E % n_group == 0,
 * k <= topk_group * E / n_group.  Returns a status.
 */
MOE_API int moe_router_topk(int32_t T, int32_t E, int32_t k, const float *logits,
                            int32_t score_fn, int32_t n_group, int32_t topk_group,
                            int32_t renormalize, int32_t *topk_idx, float *topk_w, void *stream);

/*
 * Router top-k followed by dispatch, in one call: the routing of moe_router_topk
 * on logits[T, E] (E = cfg->E, k = cfg->k) writes topk_idx[T, k] and
 * topk_w[T, k], and the dispatch of moe_dispatch reads them ("Lower latency and
 * higher throughput with multi-node DeepSeek deployment", section "Roteador
 * MoE": the router is the step right before dispatch).  Results, errors and
 * the handle are those of the two calls made one after the other.
 *
 * The router and the dispatch are two stream-ordered launches.  At decode
 * sizes (no MOE_PAD128, k <= 8, T below the SM count: the one-token-per-CTA
 * dispatch) the dispatch kernel starts while the router runs and loads and
 * quantises its rows before it waits for the router, so only the work that
 * needs the expert ids (a few KB, read from L2) follows the router.
 * workspace is moe_dispatch's (moe_workspace_bytes(cfg, T)).  Every argument
 * of both steps is checked before anything is enqueued.
 */
MOE_API int moe_route_dispatch(const moe_config *cfg, int32_t T, const void *x,
                               const float *logits, int32_t score_fn, int32_t n_group,
                               int32_t topk_group, int32_t renormalize, int32_t *topk_idx,
                               float *topk_w, const moe_dispatch_out *out, int32_t *slot,
                               void *workspace, size_t workspace_bytes, int32_t *dev_err,
                               void *stream, moe_handle *handle);

/*
 * Expert parallelism across W GPUs ("Enabling trillion-parameter models on AWS
 * EFA", sections "Buffers de Envio e Recebimento" and "Despacho e Combinação":
 * the ranks share their per-expert counts first, and each sender then writes
 * its rows into every peer's receive buffer at a range it computes itself).
 * cfg->E is the global expert count and cfg->R the number of ranks W (at most
 * 64, dividing E); rank d hosts experts [d*E/W, (d+1)*E/W).  Rank d's receive
 * buffer holds, expert by expert, the rows from rank 0, then rank 1, ..., each
 * in (token, k) order, each expert padded to 128 rows with MOE_PAD128: the
 * single-GPU layout of all ranks' batches concatenated in rank order, from
 * rank d's rank offset on.  Every rank calls, on its own stream:
 *   1. moe_dispatch_layout with R = 1 and no padding on its own batch (its
 *      counts, offsets and slots);
 *   2. an all-gather of the E counts into counts_all[W, E] (the caller's
 *      collective, e.g. NCCL);
 *   3. moe_ep_layout, then moe_ep_dispatch_payload with the W receive buffers
 *      and the "rows" flags, then moe_ep_wait on its own "rows" flags: the
 *      rank's buffer then holds every sender's rows;
 *   4. after its experts wrote their outputs, moe_ep_signal on the "outputs"
 *      flags, then moe_ep_wait on its own "outputs" flags, then moe_ep_combine
 *      with the W expert outputs.
 * No step blocks the host, so a layer's exchange can be captured in a CUDA
 * graph (section "Despacho e Combinação": a receiver uses its buffers once the
 * senders have signalled completion).
 * Buffer tables are host arrays of W device pointers (peer mappings; the
 * rank's own buffer at its index), each 16-byte aligned, every buffer
 * [rows_cap, H] (and [rows_cap, H/128] scales for fp8).  The kernels use plain
 * loads and stores, so peer memory works as local memory does.
 *
 * moe_ep_rows_capacity: the rows one rank's buffer needs when every rank
 * dispatches up to T tokens (all entries to one rank), or -1 on bad arguments.
 *
 * moe_ep_layout: from this rank's routing, its one-rank layout (local_slot
 * [T,k], local_offset [E+1]) and counts_all [W,E] (device), writes dst_row
 * [T,k] (the entry's row in the buffer of the rank hosting its expert; -1 for
 * a bad id, and -1 with MOE_DEV_CAPACITY where the row is past rows_cap),
 * recv_count [E/W] (this rank's experts' totals over all ranks) and recv_offset
 * [E/W+1] (their offsets in this rank's buffer).
 *
 * moe_ep_dispatch_payload: copies (bf16) or quantises (MOE_FP8, as
 * moe_dispatch does) x[t] into row dst_row[t,j] of the buffer of the rank that
 * hosts topk_idx[t,j].  Rows outside [-1, rows_cap) set MOE_DEV_BAD_SLOT and are
 * skipped.  With peer_flags non-NULL (a host table of W device pointers, each
 * rank's "rows" flags: W int32 per rank, zero before the first layer), the
 * kernel's last CTA, once every CTA's stores are visible at system scope,
 * increments *epoch (an int32 in this rank's memory, zero before the first
 * layer) and stores the new value into peer_flags[d][rank] of every rank d,
 * with release semantics at system scope; *done_count (an int32 in this
 * rank's memory, zero before the first layer) counts the finished CTAs and is
 * left at zero.  It signals with T = 0 too.
 *
 * moe_ep_signal: once the previous kernel in the stream has completed,
 * increments *epoch and stores it into peer_flags[d][rank] for every rank d
 * (release, system scope): the same signal without a payload, for the
 * "outputs" event after the experts.
 *
 * moe_ep_wait: waits until flags[s] >= *epoch for every sender s < W (flags
 * and epoch in this rank's memory; acquire loads at system scope, wrap-safe
 * comparison) for at most limit_ns (1 ns .. MOE_EP_MAX_WAIT_NS) in all; on
 * expiry it sets MOE_DEV_TIMEOUT in *dev_err and returns, so the stream goes
 * on and the caller learns of it from moe_check.  Kernels after it in the
 * stream see every waited-for sender's writes.
 *
 * moe_ep_combine: y[t] = bf16(sum_j w[t,j] * row dst_row[t,j] of the expert
 * output of the rank hosting topk_idx[t,j]), the fp32 chain of moe_combine.
 *
 * All return a status; argument errors enqueue nothing.
 */
MOE_API int64_t moe_ep_rows_capacity(const moe_config *cfg, int32_t T);
MOE_API int moe_ep_layout(const moe_config *cfg, int32_t rank, int32_t T, const int32_t *topk_idx,
                          const int32_t *local_slot, const int32_t *local_offset,
                          const int32_t *counts_all, int64_t rows_cap, int32_t *dst_row,
                          int32_t *recv_count, int32_t *recv_offset, int32_t *dev_err,
                          void *stream);
MOE_API int moe_ep_dispatch_payload(const moe_config *cfg, int32_t T, const void *x,
                                    const int32_t *topk_idx, const int32_t *dst_row,
                                    void *const *peer_recv_x, float *const *peer_recv_scale,
                                    int64_t rows_cap, int32_t rank, int32_t *const *peer_flags,
                                    int32_t *epoch, int32_t *done_count, int32_t *dev_err,
                                    void *stream);
MOE_API int moe_ep_signal(int32_t W, int32_t rank, int32_t *const *peer_flags, int32_t *epoch,
                          void *stream);
MOE_API int moe_ep_wait(int32_t W, const int32_t *flags, const int32_t *epoch, uint64_t limit_ns,
                        int32_t *dev_err, void *stream);
MOE_API int moe_ep_combine(const moe_config *cfg, int32_t T, const int32_t *topk_idx,
                           const int32_t *dst_row, const float *topk_w,
                           const void *const *peer_expert_out, int64_t rows_cap, void *y,
                           int32_t *dev_err, void *stream);

/*
 * moe_dispatch without a workspace argument, for callers that cannot allocate
 * device memory (the pages have no counterpart; this is a deployment aid).
 *
 * Some callers may not call cudaMalloc or any allocator: code that runs while
 * a stream is being captured into a CUDA graph, serving loops with a memory
 * plan fixed at start-up, and plain C hosts that are only handed device
 * pointers.  This entry point takes the same inputs and caller-allocated
 * outputs as moe_dispatch and computes the same results, but its metadata
 * scratch is a fixed MOE_NO_ALLOC_SCRATCH_BYTES array inside the library
 * (device memory that every GPU which loads the library holds until the
 * process exits).  It allocates nothing and frees nothing.
 *
 * - Limit: the tiled metadata needs ceil(T*k/1024) * E int32 words
 *   (moe_workspace_bytes); beyond MOE_NO_ALLOC_SCRATCH_BYTES the call returns
 *   MOE_ERR_TOO_LARGE and enqueues nothing.  With E = 256 that allows T*k up
 *   to 1,048,576 entries; with E = 2048, up to 131,072.
 * - Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current.  Make that first call
 *   before capturing any stream.
 * - Sharing: every call on a device uses the same array and leaves its
 *   contents behind; the kernels overwrite every word they read, so nothing
 *   needs clearing.  Calls whose work overlaps on the GPU (different streams
 *   with no ordering between them) race on the array and must not be made.
 */
MOE_API int moe_dispatch_no_alloc(const moe_config *cfg, int32_t T, const void *x,
                                  const int32_t *topk_idx, const float *topk_w,
                                  const moe_dispatch_out *out, int32_t *slot, int32_t *dev_err,
                                  void *stream, moe_handle *handle);

/*
 * Diagnostic of the library's bounded device waits.  Launches one warp that
 * waits on a shared-memory barrier nothing ever completes, using the same wait
 * as the bulk-copy kernels, and gives up after limit_ns nanoseconds
 * (1..1e9); it then ORs MOE_DEV_TIMEOUT into *dev_err (device pointer) and
 * returns, leaving the context usable.  Every wait in the dispatch kernels has
 * a 1 s limit and reports the same bit.  Returns a status; the bit is read with
 * moe_check.
 */
MOE_API int moe_selftest_bounded_wait(int32_t *dev_err, uint64_t limit_ns, void *stream);

/*
 * Waits for `stream`, reads the device error word, clears it (stream-ordered),
 * and stores it in *bits_out when not NULL.  Returns MOE_OK if it was 0,
 * MOE_ERR_DEVICE if not, MOE_ERR_CUDA if the stream failed.
 */
MOE_API int moe_check(int32_t *dev_err, void *stream, int32_t *bits_out);

/* Short English text for a status code. */
MOE_API const char *moe_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
MOE_API int moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DISPATCH_COMBINE_H */
