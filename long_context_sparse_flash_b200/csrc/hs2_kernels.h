// hs2_kernels.h -- host-side launchers of the libhs2 kernels (internal).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "hs2_common.cuh"

namespace hs2 {

// A validated problem, as the kernels see it.
struct Problem {
    int B, nq, hq, hkv, D, window, topk;
    int64_t q_pos0, kv_len;   // kv_len is also the row stride of k/v per (b, g)
    float scale_log2;         // softmax_scale * log2(e)
    const int64_t* seq_len;   // decode: per-sequence cache lengths (device) or nullptr
    WsHeader* err;            // device error word or nullptr
};

// count of kernel launches issued by the library
void count_launch(int n = 1);

// Per-kernel timing (enabled by hs2_profile_start): an event pair recorded on
// the launching stream around every launch.  Bracket each launch with
// prof_begin / prof_end; both are no-ops while profiling is off.
void prof_begin(uint32_t kid, cudaStream_t st);
void prof_end(cudaStream_t st);

// K0: KV bridging -- kv = hidden W_kv^T written as bf16 into k_cache / v_cache
// rows pos_b + i (see hs2_kv_bridge in hs2.h); err may be null.  With `part`
// (bridge_split_bytes(...) bytes, or null) a call with few tokens splits d_model
// over more CTAs and sums the fp32 partials in a second kernel.
int bridge_splits(int64_t n_rows, int d_model, int h_kv, int head_dim);
size_t bridge_split_bytes(int64_t n_rows, int d_model, int h_kv, int head_dim);
cudaError_t launch_bridge(int64_t n_rows, int n_new, int d_model, int h_kv, int head_dim, int64_t pos0,
                          int64_t kv_cap, const int64_t* seq_pos, const void* hidden, const void* w_kv,
                          void* k_cache, void* v_cache, WsHeader* err, cudaStream_t st, float* part = nullptr);

// K1 on tcgen05/TMEM/TMA (prefill-shaped calls: 128-row query tiles).  When
// full_tc_splits(p) > 1 and `scratch` holds full_tc_split_scratch_bytes(p),
// each CTA's key range is split and the parts merged exactly; otherwise no
// scratch is used.
int full_tc_splits(const Problem& p);
size_t full_tc_split_scratch_bytes(const Problem& p);
cudaError_t launch_full_tc(const Problem& p, const void* q, const void* k, const void* v, void* out,
                           float* lse, void* scratch, size_t scratch_bytes, cudaStream_t st);

// K1: causal full attention + LSE for every query of the call (scratch: see
// launch_full_tc; may be null).
cudaError_t launch_full(const Problem& p, const void* q, const void* k, const void* v, void* out,
                        float* lse, void* scratch, size_t scratch_bytes, cudaStream_t st);

// K2 part 1: selection scores of queries [i_begin, i_begin + i_count) into
// scores[((b * hkv + g) * i_count + (i - i_begin)) * sstride + j], j <= t - window.
cudaError_t launch_score(const Problem& p, const void* q, const void* k, const float* lse,
                         float* scores, int i_begin, int i_count, int64_t sstride,
                         cudaStream_t st);

// K2 part 2: exact top-k per (query, KV head) over the stored scores.
cudaError_t launch_topk(const Problem& p, const float* scores, int64_t sstride, int32_t* idx,
                        int i_begin, int i_count, cudaStream_t st);

// K2 on tcgen05 for prefill-shaped calls: sampled threshold, filtered sweep
// with on-chip survivor lists, exact final top-k, retry of underestimated rows.
size_t select_tc_scratch_bytes(const Problem& p, int i_count, int64_t n_cand_max);
// Byte offset, inside that scratch, of the per-row retry marks (int32, one per
// (sequence, KV head, query) row of the chunk; non-zero after the call = the
// row ran the retry pass).
size_t select_tc_status_offset(const Problem& p, int i_count, int64_t n_cand_max);
// Decode selection over few, long rows: each row cut into key chunks (each
// chunk's exact top-K with scores on its own CTA, then a per-row merge);
// chunk_scratch holds topk_chunk_bytes(p, n_cand_max) bytes (0: one CTA per row).
size_t topk_chunk_bytes(const Problem& p, int64_t n_cand_max);
cudaError_t launch_topk_decode(const Problem& p, const float* scores, int64_t sstride, int64_t n_cand_max,
                               int32_t* idx, void* chunk_scratch, cudaStream_t st);
// Block-level selection (blocks of `blk` in {32, 64, 128} keys): the chunk-sum
// sweep over the tensor cores, then the per-row block top-k.  Scratch: the
// chunk sums, block_tc_scratch_bytes(p, i_count, n_cand_max) bytes.
size_t block_tc_scratch_bytes(const Problem& p, int i_count, int64_t n_cand_max);
// Queries per CTA of the tensor-core sweeps (token and block) over rows of up
// to n_cand_max candidates with G query heads per KV head; the sweeps run one
// CTA per SM.
int select_tc_qt(int64_t n_cand_max, int G);
cudaError_t launch_block_select_tc(const Problem& p, const void* q, const void* k, const float* lse, int32_t* idx,
                                   void* scratch, int i_begin, int i_count, int64_t n_cand_max, int blk,
                                   cudaStream_t st);
cudaError_t launch_select_tc(const Problem& p, const void* q, const void* k, const float* lse, int32_t* idx,
                             void* scratch, int i_begin, int i_count, int64_t n_cand_max, cudaStream_t st,
                             float* sel_score = nullptr);

// Decode (one query per sequence): split-KV partial attention that also stores
// the candidates' logits, exact combine -> out/lse, and (scores != nullptr)
// the selection scores [B][H_kv][sstride] for the radix top-k.
size_t decode_scratch_bytes(const Problem& p);
cudaError_t launch_decode(const Problem& p, const void* q, const void* k, const void* v, void* out, float* lse,
                          void* scratch, float* scores, int64_t sstride, cudaStream_t st);

// K3: one sparse KV-reuse layer.
// with_window = 0 attends to the selected rows alone; lse (nullable) receives
// the natural-log LSE of the attended logits per (sequence, head, query).
cudaError_t launch_sparse(const Problem& p, const void* q, const void* k, const void* v,
                          const int32_t* idx, void* out, cudaStream_t st, int with_window = 1,
                          float* lse = nullptr);

// Context parallelism (cp_kernels.cu): the merges of per-slice results.
//   launch_cp_combine: P partial (out bf16 [P][rows][D], natural-log lse [P][rows])
//     -> out, lse over the union of the slices' keys;
//   launch_cp_select_merge: P per-slice top-K lists (local rows [P][rows][K],
//     ascending, -1 padded; scores [P][rows][K]) with the slices' first keys
//     offs[P] (ascending, host array) -> the whole-context top-K, ascending;
//   launch_cp_idx_local: whole-context idx -> the rows in [off, off + len),
//     shifted by -off, in order, -1 padded.
int cp_max_parts();
cudaError_t launch_cp_combine(int n_parts, int64_t rows, int head_dim, const void* out_parts, const float* lse_parts,
                              void* out, float* lse, cudaStream_t st);
cudaError_t launch_cp_select_merge(int n_parts, int64_t rows, int topk, const int32_t* idx_parts,
                                   const float* score_parts, const int64_t* offs, int32_t* idx, cudaStream_t st);
cudaError_t launch_cp_idx_local(int64_t rows, int topk, const int32_t* idx, int64_t off, int64_t len, int32_t* out,
                                cudaStream_t st);

// Query position of query 0 of sequence b: q_pos0, or seq_len[b] - nq for decode
// (clamped into [0, kv_len - nq]; a clamp is reported through the error word).
__device__ __forceinline__ int64_t seq_pos0(const Problem& p, int b, uint32_t kid) {
    if (p.seq_len == nullptr) return p.q_pos0;
    int64_t len = p.seq_len[b];
    if (len < p.nq || len > p.kv_len) {
        if (threadIdx.x == 0) report_error(p.err, HS2_ERR_DEVICE_CHECK, kid, (uint32_t)b, (uint32_t)len);
        len = len < p.nq ? p.nq : p.kv_len;
    }
    return len - p.nq;
}

}  // namespace hs2
