/*
 * hs2.h -- C ABI of libhs2: HySparse2 Cross-Decoder attention on one B200.
 *
 * The method (HySparse2 pages):
 *   - xiawanshe.com report, section "两级KV共享" (second level, "KV Reuse"):
 *     inside the Cross-Decoder one full-attention layer produces the KV cache
 *     and a token-selection result, and several following sparse-attention
 *     layers reuse both.
 *   - same report, section "Token级选择": selection is per token, anywhere in
 *     the context; the separate SWA branch is dropped; the most recent 128
 *     tokens are always attended and 1024 tokens are selected from the older
 *     context; local and global attention share one KV cache.
 *   - davidyin.dev video notes, section "HySparse2 的解法": no extra indexer
 *     is trained for the selection.
 *
 * Definitions used by every entry point (t = absolute position of a query):
 *   s_{h,j}   = softmax_scale * <q_h, k_{g,j}>, g = h / G, G = h_q / h_kv, j in [0, t]
 *   lse_h     = ln sum_{j<=t} exp(s_{h,j})            (natural log, fp32)
 *   out_h     = sum_{j<=t} exp(s_{h,j} - lse_h) v_{g,j}
 *   window(t) = [max(0, t-window+1), t]               (window tokens incl. t)
 *   score_{g,j} = sum_{h in g} exp(s_{h,j} - lse_h),   j in [0, t-window]
 *   idx_g(t)  = the min(topk, max(0, t-window+1)) candidates first in the order
 *               (score descending, j ascending), stored ascending by j, then
 *               -1 padding up to topk entries.
 *   sparse layer: out'_h = softmax over S = idx_g(t) U window(t) of
 *               softmax_scale * <q'_h, k_{g,j}>, applied to v_{g,j}.
 *
 * Layouts (all row-major, contiguous, device memory, 16-byte aligned):
 *   q, q'  [batch, h_q, n_q, head_dim]      bf16
 *   k, v   [batch, h_kv, kv_len, head_dim]  bf16   (the shared cache)
 *   out    [batch, h_q, n_q, head_dim]      bf16
 *   lse    [batch, h_q, n_q]                fp32
 *   idx    [batch, h_kv, n_q, topk]         int32
 * Query i of a call sits at t = q_pos0 + i; kv_len >= q_pos0 + n_q.
 *
 * Ownership: the caller allocates and owns every buffer, including the
 * workspace; the library allocates no device memory and keeps no per-call
 * state, with one exception: the static device array behind
 * hs2_full_attn_select_static (HS2_STATIC_SCRATCH_BYTES, held on every GPU
 * that loads the library until the process exits).  Execution: every entry point validates its arguments on the host,
 * returns an error status without launching anything if a check fails, and
 * otherwise enqueues its kernels on `stream` and returns at once (no host
 * synchronisation), except hs2_get_device_status which synchronises `stream`.
 * A call whose sizes make the work empty (batch == 0 or n_q == 0) returns
 * HS2_OK without launching.
 */
#ifndef HS2_H
#define HS2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Binary compatible with cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* hs2_stream_t;

typedef enum {
    HS2_OK = 0,
    HS2_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer      */
    HS2_ERR_UNSUPPORTED = 2,   /* valid but outside the built kernels' range      */
    HS2_ERR_WORKSPACE = 3,     /* ws_bytes below hs2_workspace_size()             */
    HS2_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed            */
    HS2_ERR_DEVICE_CHECK = 5,  /* a kernel found an invalid input (error word)    */
    HS2_ERR_TIMEOUT = 6        /* a bounded device-side wait gave up (error word) */
} hs2_status;

/* Problem description shared by all entry points.
 *   head_dim in {64, 128}; h_q % h_kv == 0 with G = h_q / h_kv in {1, 2, 4, 8};
 *   1 <= window <= 1024; 0 <= topk <= 2048; q_pos0 >= 0;
 *   q_pos0 + n_q <= kv_len <= 2^31 - 1; softmax_scale == 0 selects 1/sqrt(head_dim),
 *   otherwise it must be finite and > 0; reserved must be 0. */
typedef struct {
    int32_t batch;
    int32_t n_q;
    int32_t h_q;
    int32_t h_kv;
    int32_t head_dim;
    int32_t window;
    int32_t topk;
    int32_t reserved;
    int64_t q_pos0;
    int64_t kv_len;
    float softmax_scale;
} hs2_shape;

enum {
    HS2_ENTRY_FULL_SELECT = 0,
    HS2_ENTRY_SPARSE = 1,
    HS2_ENTRY_PREFILL = 2,
    HS2_ENTRY_DECODE = 3,
    HS2_ENTRY_BLOCK_SELECT = 4,
    HS2_ENTRY_CP_ATTN = 5,     /* slice calls: sized by hs2_cp_workspace_size */
    HS2_ENTRY_CP_SELECT = 6,
    HS2_ENTRY_CP_SPARSE = 7
};

/* Bytes of workspace the entry point `entry` needs for `shape` (0 if the shape
 * is invalid, and 0 for the context-parallel slice entries, which
 * hs2_cp_workspace_size sizes).  The first 256 bytes of every workspace hold
 * the device error word; hs2_workspace_init() must zero them once before first
 * use. */
size_t hs2_workspace_size(const hs2_shape* shape, int entry);

/* Zero the workspace header (error word) on `stream`.  Asynchronous. */
hs2_status hs2_workspace_init(void* ws, size_t ws_bytes, hs2_stream_t stream);

/* Full-attention layer of the Cross-Decoder with token selection
 * (xiawanshe.com report, "两级KV共享" KV Reuse + "Token级选择").
 * Reads q, k, v; writes out, lse and idx for every query of the call.  Runs the
 * full-attention pass, then the selection pass that recomputes the scores
 * from the written LSE (two separate kernels).  ws: hs2_workspace_size(shape,
 * HS2_ENTRY_FULL_SELECT) bytes, contents are scratch except the header. */
hs2_status hs2_full_attn_select(const hs2_shape* shape, const void* q, const void* k,
                                const void* v, void* out, float* lse, int32_t* idx,
                                void* ws, size_t ws_bytes, hs2_stream_t stream);

/* One sparse KV-reuse layer (xiawanshe.com report, "两级KV共享": the following
 * sparse layers reuse the full layer's cache and selection; "Token级选择": they
 * attend to the selected tokens plus the forced recent window).  q is this
 * layer's own query; k, v and idx are those of the full-attention layer.
 * idx rows must be as hs2_full_attn_select writes them (ascending valid
 * entries in [0, t-window], then -1); the checked build reports violations
 * through the error word.  ws may be NULL with ws_bytes == 0. */
hs2_status hs2_sparse_attn(const hs2_shape* shape, const void* q, const void* k, const void* v,
                           const int32_t* idx, void* out, void* ws, size_t ws_bytes,
                           hs2_stream_t stream);

/* The full-attention layer with BLOCK-level selection at the same budget, the
 * design token-level selection replaces (xiawanshe.com report, section
 * "Token级选择": the earlier HySparse chose whole blocks of contiguous tokens).
 * Same arguments, layouts and outputs as hs2_full_attn_select (any q_pos0, so
 * it also serves prefill chunks), plus the block size.  Definitions:
 *   block bb = keys [bb*block, (bb+1)*block), block in {32, 64, 128};
 *   candidate blocks: those lying wholly in [0, t-window], n_blk(t) =
 *   (t-window+1) / block of them (a partial block next to the window is not a
 *   candidate);
 *   block score = sum of score_{g,j} over the block's keys;
 *   idx_g(t) = the keys of the first min(topk / block, n_blk) blocks in the
 *   order (block score descending, bb ascending), stored ascending, then -1
 *   padding up to topk entries.
 * Any other block size returns HS2_ERR_UNSUPPORTED.  ws:
 * hs2_workspace_size(shape, HS2_ENTRY_BLOCK_SELECT) bytes.  The output feeds
 * hs2_sparse_attn unchanged. */
hs2_status hs2_full_attn_block_select(const hs2_shape* shape, int32_t block, const void* q, const void* k,
                                      const void* v, void* out, float* lse, int32_t* idx, void* ws,
                                      size_t ws_bytes, hs2_stream_t stream);

/* The two attention branches of a sparse layer in the predecessor design, as
 * a cost comparator for hs2_sparse_attn (xiawanshe.com report, section
 * "Token级选择": HySparse2 drops the Cross-Decoder's separate sliding-window
 * branch and keeps the most recent tokens in the one shared cache instead).
 * Per query t and head h (g = h / G), with the layer's own query q:
 *   window branch:   out_swa, lse_swa = softmax attention over window(t) of the
 *                    branch's OWN cache k_swa, v_swa ([batch, h_kv, kv_len,
 *                    head_dim] bf16, laid out like k, v);
 *   selected branch: out_sel, lse_sel = softmax attention over the selected
 *                    rows idx_g(t) ALONE (no window) of the shared cache k, v;
 *                    a row with no selected key gets out_sel = 0 and
 *                    lse_sel = -inf.
 * out_* [batch, h_q, n_q, head_dim] bf16; lse_* [batch, h_q, n_q] fp32,
 * natural log.  The pages do not say how the predecessor combined the two
 * outputs, so both are returned; merging them by their LSEs gives the softmax
 * over idx U window.  idx rows as hs2_sparse_attn takes them (topk = 0 makes
 * the selected branch empty).  ws may be NULL with ws_bytes == 0; with a
 * workspace, the checked build reports invalid idx rows through its error
 * word.  Two kernel launches (kernel id 4 each). */
hs2_status hs2_swa_branches(const hs2_shape* shape, const void* q, const void* k_swa, const void* v_swa,
                            const void* k, const void* v, const int32_t* idx, void* out_swa, float* lse_swa,
                            void* out_sel, float* lse_sel, void* ws, size_t ws_bytes, hs2_stream_t stream);

/* ---------------------------------------------------------------------------
 * Context parallelism: the KV cache of one long context is cut into P
 * contiguous slices, slice p holding keys [kv_off_p, kv_off_p + len_p) on its
 * own GPU (offsets ascending, slices adjacent).  The layers of the pages
 * (xiawanshe.com report, sections "两级KV共享" and "Token级选择") are computed
 * exactly, with one exchange of per-slice results after each step:
 *   1. hs2_cp_attn_partial on every slice -> out_p, lse_p (attention over the
 *      slice's causal keys); exchange; hs2_cp_combine -> out, lse.
 *   2. hs2_cp_select_local on every slice with the combined lse -> the slice's
 *      top-K candidates and their scores; exchange; hs2_cp_select_merge -> idx
 *      (the same rows hs2_full_attn_select selects from the whole cache).
 *   3. per sparse layer: hs2_cp_sparse_partial on every slice -> out_p, lse_p
 *      (the layer over the rows of idx U window the slice holds); exchange;
 *      hs2_cp_combine -> out.
 * The exchange itself (an all-gather of the per-slice buffers, stacked along
 * a new leading axis in slice order) is the caller's; the library only
 * computes.  Slice calls take a `shape` describing the slice: kv_len = len_p
 * rows (the row stride of k, v), q_pos0 = the ABSOLUTE position of query 0
 * (any q_pos0 >= 0: a query may sit before the slice -- it has no key there,
 * out_p = 0 and lse_p = -inf -- or after it -- every key of the slice is
 * causal for it); n_q >= 64 (HS2_ERR_UNSUPPORTED below).  Candidates are still
 * the keys j <= t - window in absolute positions.  Slice calls need a
 * workspace of hs2_cp_workspace_size(shape, kv_off, entry) bytes. */

/* Bytes of workspace a slice call needs (0 if the shape or entry is invalid). */
size_t hs2_cp_workspace_size(const hs2_shape* shape, int64_t kv_off, int entry);

/* Step 1 on one slice: out [batch, h_q, n_q, head_dim] bf16 and lse [batch,
 * h_q, n_q] fp32 (natural log) of the attention over the slice's keys
 * j <= t.  Entry HS2_ENTRY_CP_ATTN. */
hs2_status hs2_cp_attn_partial(const hs2_shape* shape, int64_t kv_off, const void* q, const void* k, const void* v,
                               void* out, float* lse, void* ws, size_t ws_bytes, hs2_stream_t stream);

/* Step 2 on one slice: with lse the COMBINED (whole-context) LSE, the slice's
 * top-min(topk, its candidates) keys by (score desc, j asc): idx [batch,
 * h_kv, n_q, topk] int32 as LOCAL rows of the slice (ascending, -1 padded) and
 * score [batch, h_kv, n_q, topk] fp32 (the group-summed probability, -1 for
 * padding).  Entry HS2_ENTRY_CP_SELECT. */
hs2_status hs2_cp_select_local(const hs2_shape* shape, int64_t kv_off, const void* q, const void* k,
                               const float* lse, int32_t* idx, float* score, void* ws, size_t ws_bytes,
                               hs2_stream_t stream);

/* Step 3 on one slice: one sparse layer (q its own query) over the rows of
 * idx U window(t) that the slice holds; idx is the whole-context selection
 * (absolute rows, as hs2_cp_select_merge writes it).  out bf16, lse fp32
 * (natural log; -inf and out = 0 for a query with no such row in the slice).
 * Entry HS2_ENTRY_CP_SPARSE. */
hs2_status hs2_cp_sparse_partial(const hs2_shape* shape, int64_t kv_off, const void* q, const void* k,
                                 const void* v, const int32_t* idx, void* out, float* lse, void* ws, size_t ws_bytes,
                                 hs2_stream_t stream);

/* The merge of steps 1 and 3: out_parts [n_parts][n_rows][head_dim] bf16 and
 * lse_parts [n_parts][n_rows] fp32 (n_rows = batch * h_q * n_q) -> out, lse:
 * lse = ln sum_p e^(lse_p), out = sum_p e^(lse_p - lse) out_p; a row whose parts
 * are all -inf gets 0 and -inf.  Device buffers; stream-ordered. */
hs2_status hs2_cp_combine(int32_t n_parts, int64_t n_rows, int32_t head_dim, const void* out_parts,
                          const float* lse_parts, void* out, float* lse, hs2_stream_t stream);

/* The merge of step 2: shape is the WHOLE context's (kv_len = total keys, the
 * usual q_pos0 rule); kv_offs is a HOST array of the n_parts slices' first keys
 * (strictly ascending; n_parts <= 16); idx_parts / score_parts stack the
 * slices' hs2_cp_select_local outputs in slice order.  Writes idx [batch, h_kv,
 * n_q, topk]: the whole-context selection, absolute rows ascending, -1 padded. */
hs2_status hs2_cp_select_merge(const hs2_shape* shape, int32_t n_parts, const int64_t* kv_offs,
                               const int32_t* idx_parts, const float* score_parts, int32_t* idx,
                               hs2_stream_t stream);

/* Prefill-chunk entry: the full-attention + selection layer for a chunk of
 * n_q new tokens appended to a cache of kv_len tokens (q_pos0 = kv_len - n_q
 * for an append; any q_pos0 with q_pos0 + n_q <= kv_len is accepted).  Same
 * arguments, workspace rule and outputs as hs2_full_attn_select. */
hs2_status hs2_prefill_chunk(const hs2_shape* shape, const void* q, const void* k,
                             const void* v, void* out, float* lse, int32_t* idx, void* ws,
                             size_t ws_bytes, hs2_stream_t stream);

/* Decode entry: one new token per sequence (n_q == 1).  kv_len_per_seq is a
 * device array of `batch` int64 lengths (1 <= len <= kv_len; the query of
 * sequence b sits at t = len_b - 1 and its own K/V row is already in the
 * cache), or NULL for len_b = kv_len for every b (q_pos0 is then ignored).
 * The selection pass splits every sequence's candidates over many CTAs.
 * Out-of-range lengths are clamped and reported through the error word. */
hs2_status hs2_decode(const hs2_shape* shape, const int64_t* kv_len_per_seq, const void* q,
                      const void* k, const void* v, void* out, float* lse, int32_t* idx,
                      void* ws, size_t ws_bytes, hs2_stream_t stream);

/* One sparse KV-reuse layer for decode-shaped calls (n_q == 1) whose sequences
 * have their own cache lengths: the query of sequence b sits at
 * t = kv_len_per_seq[b] - 1 (device int64 array; NULL means kv_len for every
 * b).  Otherwise identical to hs2_sparse_attn; idx is what hs2_decode wrote. */
hs2_status hs2_decode_sparse(const hs2_shape* shape, const int64_t* kv_len_per_seq, const void* q,
                             const void* k, const void* v, const int32_t* idx, void* out, void* ws,
                             size_t ws_bytes, hs2_stream_t stream);

/* Bytes of the static scratch array behind hs2_full_attn_select_static. */
#define HS2_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* hs2_full_attn_select for callers that cannot allocate device memory at the
 * point where they run the layer: a process whose device memory is a
 * pre-sized pool it may not grow, a host runtime or plugin that hands over
 * only the input and output buffers, or a step that must not synchronise the
 * device (cudaMalloc and cudaFree may).  The HySparse2 pages have no
 * counterpart for it: it is a deployment convenience, not part of the method.
 *
 * Arguments and outputs are those of hs2_full_attn_select without the
 * workspace.  Instead of a caller workspace it uses one static device array
 * of HS2_STATIC_SCRATCH_BYTES inside the library; every GPU that loads the
 * library holds that array until the process exits.  Calls no allocation
 * routine.  Shapes whose workspace (hs2_workspace_size(shape,
 * HS2_ENTRY_FULL_SELECT)) exceeds HS2_STATIC_SCRATCH_BYTES are rejected with
 * HS2_ERR_WORKSPACE before anything is launched; invalid shapes get the
 * status hs2_full_attn_select would give.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and keeps it for the life
 * of the process; make that first call before any stream capture, and do not
 * use this entry point across a cudaDeviceReset (or any teardown of the
 * device's primary context): the kept address would then be stale.  Every
 * call first clears the error-word header of the array on `stream` (the array
 * keeps the previous call's contents); hs2_static_scratch_status reads what
 * the last call reported.  All calls on a device share the one array: calls
 * that overlap on the GPU (other streams, or other host threads without
 * ordering) race on it and corrupt each other's selections; order them on one
 * stream or serialise them. */
hs2_status hs2_full_attn_select_static(const hs2_shape* shape, const void* q, const void* k,
                                       const void* v, void* out, float* lse, int32_t* idx,
                                       hs2_stream_t stream);

/* HS2_STATIC_SCRATCH_BYTES, for callers that load the library dynamically. */
size_t hs2_static_scratch_bytes(void);

/* The device error word of the static array, as hs2_get_device_status reads a
 * workspace's: synchronises `stream`, returns HS2_OK, HS2_ERR_DEVICE_CHECK or
 * HS2_ERR_TIMEOUT for the last hs2_full_attn_select_static call on the
 * current device (HS2_ERR_CUDA if a runtime call fails), fills info[0..4) if
 * non-NULL, and clears the word.  Copies through host stack memory; allocates
 * nothing.  Read it before the next static call, which clears the word. */
hs2_status hs2_static_scratch_status(hs2_stream_t stream, uint32_t* info);

/* Synchronise `stream`, read and clear the workspace error word.  Returns
 * HS2_OK, HS2_ERR_DEVICE_CHECK or HS2_ERR_TIMEOUT (or HS2_ERR_CUDA).  If
 * `info` is non-NULL it receives 4 words: code, kernel id, and two values
 * describing the first failure. */
hs2_status hs2_get_device_status(void* ws, hs2_stream_t stream, uint32_t* info);

/* Diagnostics: how many selection rows of the last query chunk of the last
 * hs2_full_attn_select / hs2_prefill_chunk call on this workspace ran the
 * selection's retry pass.  The selection first estimates, per (query, KV head)
 * row, a score bound that at least min(topk, candidates) candidates exceed,
 * from a fixed-stride sample of the keys; a row where fewer candidates pass is
 * marked and swept again with bound 0, which keeps the selection exact.  This
 * reads those marks: synchronises `stream`, copies them from `ws` (the call's
 * workspace, same shape) to host memory and writes their count to *n_rows (0
 * for shapes whose selection takes no sample: few candidates, n_q < 16 or
 * topk == 0).  Not part of the method (no counterpart in the paper). */
hs2_status hs2_select_retry_rows(const hs2_shape* shape, const void* ws, size_t ws_bytes, hs2_stream_t stream,
                                 int64_t* n_rows);

/* Static description of a status code. */
const char* hs2_status_string(hs2_status status);

/* Number of kernels this library has launched in this process (all threads). */
uint64_t hs2_launch_count(void);

/* Measurement aid: from hs2_profile_start() on, the library records a CUDA
 * event pair on the launching stream around every kernel it launches (event
 * objects only, no device memory).  hs2_profile_stop() ends the recording,
 * waits for the recorded events, and writes, for every kernel id u < n_kinds,
 * the summed event time in ms (total_ms[u]) and the launch count
 * (launches[u]); either array may be NULL.  Kernel ids: 1 full attention,
 * 2 selection scores, 3 top-k select, 4 sparse attention, 5 decode attention
 * partials, 6 decode combine, 7 fused attention + selection, 8 selection
 * threshold estimate, 9 filtered selection sweep, 10 selection retry,
 * 11 KV bridging, 12 block-selection score sweep, 13 block top-k,
 * 14 context-parallel combine, 15 context-parallel selection merge,
 * 16 context-parallel selection slicing, 17 the bounded-wait self-test. */
hs2_status hs2_profile_start(void);
hs2_status hs2_profile_stop(uint32_t n_kinds, float* total_ms, uint64_t* launches);

/* Diagnostics: evaluate the library's exp2 implementations at n device points
 * x: y[0..n) = hardware ex2, y[n..2n) = degree-3 polynomial, y[2n..3n) =
 * degree-5 polynomial, y[3n..4n) and y[4n..5n) = the two-lane packed degree-5
 * form at (x, x/2) (the FMA-pipe 2^x used beside the hardware unit in the
 * softmax and selection kernels).  y holds 5n floats.  Asynchronous on
 * `stream`. */
hs2_status hs2_selftest_exp2(const float* x, float* y, int n, hs2_stream_t stream);

/* KV bridging (xiawanshe.com report, section "两级KV共享", first level "KV
 * Bridging": the Cross-Decoder's K and V are computed from the Self-Decoder's
 * hidden states).  For every new token (b, i) of the call:
 *     kv[f] = sum_c hidden[b][i][c] * w_kv[f][c],        f < 2 * h_kv * D
 *     k_cache[b][f / D][pos_b + i][f % D]        = bf16(kv[f])   f <  h_kv * D
 *     v_cache[b][f / D - h_kv][pos_b + i][f % D] = bf16(kv[f])   otherwise
 * with pos_b = seq_pos[b] (device int64 array of `batch`) or, if seq_pos is
 * NULL, pos0 for every sequence.  Only those cache rows are written (this is
 * also the decode-time cache append, n_new = 1).  fp32 accumulation, one
 * rounding to bf16 (round to nearest even).  Layouts (device, caller-owned,
 * 16-byte aligned): hidden [batch][n_new][d_model] bf16; w_kv
 * [2 * h_kv * D][d_model] bf16 (row f = output feature); k_cache, v_cache
 * [batch][h_kv][kv_cap][D] bf16.  Requires d_model > 0 a multiple of 64, D in
 * {64, 128}, h_kv * D a multiple of 256 (so each 256-feature tile lies in K
 * or in V), 0 <= pos0, pos0 + n_new <= kv_cap when seq_pos is NULL (else
 * HS2_ERR_INVALID_ARG / HS2_ERR_UNSUPPORTED).  With seq_pos, a sequence whose
 * rows would fall outside [0, kv_cap) writes nothing and is reported through
 * the error word (HS2_ERR_DEVICE_CHECK, kernel id 11).  ws: at least
 * hs2_workspace_size(..., HS2_ENTRY_SPARSE) bytes (the header), or NULL with
 * ws_bytes == 0 (then no error word).  With hs2_kv_bridge_workspace_size(shape)
 * bytes, a call with few tokens (e.g. the decode append) splits d_model over
 * more CTAs and sums fp32 partials in a second kernel (kernel id 11 too): the
 * same rows, the fp32 sum taken in another order.  Asynchronous on `stream`. */
typedef struct {
    int32_t batch;     /* sequences */
    int32_t n_new;     /* new tokens per sequence */
    int32_t d_model;   /* hidden size of the Self-Decoder */
    int32_t h_kv;      /* KV heads */
    int32_t head_dim;  /* D */
    int32_t reserved;  /* must be 0 */
    int64_t pos0;      /* cache position of token 0 when seq_pos is NULL */
    int64_t kv_cap;    /* cache rows per (sequence, head) */
} hs2_bridge_shape;
hs2_status hs2_kv_bridge(const hs2_bridge_shape* shape, const int64_t* seq_pos, const void* hidden,
                         const void* w_kv, void* k_cache, void* v_cache, void* ws, size_t ws_bytes,
                         hs2_stream_t stream);

/* Workspace bytes that enable hs2_kv_bridge's split path for `shape` (the
 * 256-byte header alone when the call has enough tokens not to need it; 0 for
 * an invalid shape). */
size_t hs2_kv_bridge_workspace_size(const hs2_bridge_shape* shape);

/* Diagnostics: the gather-bandwidth probe behind the sparse layer's roofline
 * (the sparse layer reads whole 256-byte K/V rows in data-dependent order).
 * Reads, `passes` times, the 256-byte rows rows[order[u]] (u < n_order) of
 * `rows` (device, n_rows x 256 bytes, 16-byte aligned) with 16-byte loads,
 * sixteen in flight per thread, on (SM count x 8) CTAs of 256 threads; an
 * index outside [0, n_rows) reads row 0 instead.  `sink` (device, 16 bytes, 16-byte aligned)
 * is written only in a case that keeps the loads alive and is practically never
 * taken.  The caller times the call on `stream`; bytes read = passes *
 * n_order * 256.  Requires n_order > 0, n_order % 32 == 0, passes >= 1, else
 * HS2_ERR_INVALID_ARG.  Not part of the method (no counterpart in the paper). */
hs2_status hs2_gather_probe(const void* rows, int64_t n_rows, const int32_t* order, int64_t n_order,
                            int32_t passes, void* sink, hs2_stream_t stream);

/* Diagnostics: the special-function-unit probe behind the selection sweep's
 * roofline (its binding unit is the ex2 rate: one 2^x per candidate and head).
 * Launches (SM count x 8) CTAs of 256 threads, each thread running 8
 * independent chains of `iters` hardware ex2 steps, on `stream`; writes the
 * number of ex2 executed to *ex2_count (host) at once.  `sink` (device, one
 * float) is written only in a case that practically never occurs.  The caller
 * times the call.  Requires iters >= 1 and non-null pointers, else
 * HS2_ERR_INVALID_ARG.  Not part of the method (no counterpart in the paper). */
hs2_status hs2_ex2_probe(int32_t iters, float* sink, hs2_stream_t stream, int64_t* ex2_count);

/* Diagnostics: the timeout path of the bounded device-side waits.  One CTA of
 * four warps waits, on `stream`, on an mbarrier that nothing completes, with
 * the same wait the tcgen05 kernels use but bounded by limit_cycles SM clock
 * cycles (those kernels use 2^32).  The wait gives up, the CTA's abort flag
 * releases the other warps, HS2_ERR_TIMEOUT is written into the error word of
 * `ws` (kernel id 17, a = 1, b = the reporting block) and the kernel returns:
 * hs2_get_device_status then reads HS2_ERR_TIMEOUT, and the context stays
 * usable.  ws: a workspace of ws_bytes >= 256 bytes, 256-byte aligned, owned
 * by the caller (its header is the error word; hs2_workspace_init clears it).
 * Requires 1 <= limit_cycles <= 2^32, else HS2_ERR_INVALID_ARG.  Not part of
 * the method (no counterpart in the paper). */
hs2_status hs2_selftest_wait(void* ws, size_t ws_bytes, int64_t limit_cycles, hs2_stream_t stream);

/* 1 when the library was built with device-side input checks (HS2_CHECKED). */
int hs2_is_checked_build(void);

#ifdef __cplusplus
}
#endif

#endif /* HS2_H */
