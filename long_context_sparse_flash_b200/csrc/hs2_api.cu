// hs2_api.cu -- the extern "C" boundary of libhs2: argument validation,
// workspace layout, dispatch of the kernels onto the caller's stream.
#include <atomic>
#include <cmath>
#include <mutex>
#include <vector>

#include "hs2_kernels.h"

namespace hs2 {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// ---------------------------------------------------------------------------
// per-kernel event timing (measurement aid; off unless hs2_profile_start ran)

namespace {
struct ProfRec {
    uint32_t kid;
    cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::atomic<bool> g_prof_on{false};
std::vector<ProfRec> g_prof_recs;      // recorded, not yet collected
std::vector<cudaEvent_t> g_prof_pool;  // free events
thread_local uint32_t t_prof_kid = 0;
thread_local cudaEvent_t t_prof_a = nullptr;

cudaEvent_t prof_event() {
    cudaEvent_t e = nullptr;
    if (!g_prof_pool.empty()) {
        e = g_prof_pool.back();
        g_prof_pool.pop_back();
    } else if (cudaEventCreate(&e) != cudaSuccess) {
        e = nullptr;
    }
    return e;
}
}  // namespace

void prof_begin(uint32_t kid, cudaStream_t st) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    t_prof_kid = kid;
    t_prof_a = prof_event();
    if (t_prof_a) cudaEventRecord(t_prof_a, st);
}

void prof_end(cudaStream_t st) {
    if (!g_prof_on.load(std::memory_order_relaxed) || t_prof_a == nullptr) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    cudaEvent_t b = prof_event();
    if (b) {
        cudaEventRecord(b, st);
        g_prof_recs.push_back({t_prof_kid, t_prof_a, b});
    } else {
        g_prof_pool.push_back(t_prof_a);
    }
    t_prof_a = nullptr;
}

namespace {

constexpr size_t kHeader = sizeof(WsHeader);
constexpr size_t kScoreBudget = size_t(1) << 30;  // bytes of stored scores per chunk of queries

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

// Host validation of the shape; fills `p` on success.
hs2_status check_shape(const hs2_shape* s, Problem* p) {
    if (s == nullptr) return HS2_ERR_INVALID_ARG;
    if (s->reserved != 0) return HS2_ERR_INVALID_ARG;
    if (s->batch < 0 || s->n_q < 0 || s->h_q <= 0 || s->h_kv <= 0 || s->head_dim <= 0) return HS2_ERR_INVALID_ARG;
    if (s->h_q % s->h_kv != 0) return HS2_ERR_INVALID_ARG;
    if (s->window < 1 || s->topk < 0 || s->q_pos0 < 0 || s->kv_len < 0) return HS2_ERR_INVALID_ARG;
    if (s->q_pos0 + (int64_t)s->n_q > s->kv_len) return HS2_ERR_INVALID_ARG;
    const float sc = s->softmax_scale;
    if (!(sc == 0.f || (std::isfinite(sc) && sc > 0.f))) return HS2_ERR_INVALID_ARG;
    const int G = s->h_q / s->h_kv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return HS2_ERR_UNSUPPORTED;
    if (s->head_dim != 64 && s->head_dim != 128) return HS2_ERR_UNSUPPORTED;
    if (s->window > 1024 || s->topk > 2048) return HS2_ERR_UNSUPPORTED;
    if (s->kv_len > INT32_MAX || s->batch > 65535 || s->h_q > 65535) return HS2_ERR_UNSUPPORTED;
    p->B = s->batch;
    p->nq = s->n_q;
    p->hq = s->h_q;
    p->hkv = s->h_kv;
    p->D = s->head_dim;
    p->window = s->window;
    p->topk = s->topk;
    p->q_pos0 = s->q_pos0;
    p->kv_len = s->kv_len;
    const float scale = sc == 0.f ? 1.0f / std::sqrt((float)s->head_dim) : sc;
    p->scale_log2 = scale * kLog2e;
    p->seq_len = nullptr;
    p->err = nullptr;
    return HS2_OK;
}

// Selection pass plan.  Prefill-shaped calls run the tcgen05 selection
// (sample, threshold, filtered sweep, retry) over chunks of `chunk` queries;
// decode-shaped calls store every candidate's score (sstride floats per row)
// and run the radix top-k over them.
struct ScorePlan {
    bool tc = false;
    int64_t sstride = 0;
    int64_t n_cand_max = 0;
    int chunk = 0;
    size_t bytes = 0;
};

constexpr size_t kSampleBudget = size_t(1) << 30;  // bytes of per-row selection state per chunk

ScorePlan score_plan(const Problem& p, bool decode) {
    ScorePlan sp;
    const int64_t t_hi = decode ? p.kv_len - 1 : p.q_pos0 + p.nq - 1;
    const int64_t cand = t_hi - p.window + 1;
    if (cand <= p.topk || p.nq == 0 || p.B == 0 || p.topk == 0) return sp;  // every row takes all candidates
    sp.n_cand_max = cand;
    if (!decode && p.nq >= 16) {
        sp.tc = true;
        const size_t per_q = (size_t)p.B * p.hkv * (1024 * 4 + 12);
        int64_t chunk = (int64_t)(kSampleBudget / per_q) / 32 * 32;
        if (chunk < 32) chunk = 32;
        if (chunk > p.nq) chunk = p.nq;
        sp.chunk = (int)chunk;
        sp.bytes = select_tc_scratch_bytes(p, sp.chunk, cand);
        return sp;
    }
    sp.sstride = (cand + 3) / 4 * 4;
    const size_t per_q = (size_t)p.B * p.hkv * sp.sstride * 4;
    int64_t chunk = (int64_t)(kScoreBudget / per_q);
    if (chunk >= 256) chunk = chunk / 128 * 128;
    if (chunk < 1) chunk = 1;
    if (chunk > p.nq) chunk = p.nq;
    sp.chunk = (int)chunk;
    sp.bytes = (size_t)chunk * per_q;
    return sp;
}

hs2_status cuda_status(cudaError_t e) { return e == cudaSuccess ? HS2_OK : HS2_ERR_CUDA; }

// Workspace after the header for prefill-shaped calls: the selection scratch,
// or the full layer's split parts if larger (the two are never live together).
size_t prefill_body_bytes(const Problem& p, const ScorePlan& sp) {
    const size_t split = full_tc_split_scratch_bytes(p);
    return sp.bytes > split ? sp.bytes : split;
}

hs2_status run_full_select(const hs2_shape* shape, const int64_t* seq_len, bool decode, const void* q,
                           const void* k, const void* v, void* out, float* lse, int32_t* idx, void* ws,
                           size_t ws_bytes, hs2_stream_t stream) {
    Problem p;
    hs2_status s = check_shape(shape, &p);
    if (s != HS2_OK) return s;
    if (decode && p.nq != 1 && p.nq != 0) return HS2_ERR_INVALID_ARG;
    if (p.B == 0 || p.nq == 0) return HS2_OK;
    if (!q || !k || !v || !out || !lse || !ws) return HS2_ERR_INVALID_ARG;
    if (p.topk > 0 && !idx) return HS2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
        !aligned(idx, 4) || !aligned(ws, 256) || (seq_len && !aligned(seq_len, 8)))
        return HS2_ERR_INVALID_ARG;
    const ScorePlan sp = score_plan(p, decode);
    const size_t extra = decode ? decode_scratch_bytes(p) + topk_chunk_bytes(p, sp.n_cand_max) : 0;
    const size_t body = decode ? (sp.bytes + 255) / 256 * 256 + extra : prefill_body_bytes(p, sp);
    if (ws_bytes < kHeader + body) return HS2_ERR_WORKSPACE;
    p.seq_len = seq_len;
    p.err = reinterpret_cast<WsHeader*>(ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (decode) {
        // split-KV attention (+ stored logits) -> combine -> scores -> exact top-k
        float* scores = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + kHeader);
        void* scratch = reinterpret_cast<uint8_t*>(ws) + kHeader + (sp.bytes + 255) / 256 * 256;
        const bool sel = p.topk > 0 && sp.sstride > 0;
        cudaError_t e = launch_decode(p, q, k, v, out, lse, scratch, sel ? scores : nullptr, sp.sstride, st);
        if (e != cudaSuccess) return HS2_ERR_CUDA;
        if (p.topk == 0) return HS2_OK;
        // the chunk lists of the selection sit after the decode attention's scratch
        void* chunk = topk_chunk_bytes(p, sp.n_cand_max) > 0
                          ? reinterpret_cast<uint8_t*>(scratch) + decode_scratch_bytes(p)
                          : nullptr;
        e = sel ? launch_topk_decode(p, scores, sp.sstride, sp.n_cand_max, idx, chunk, st)
                : launch_topk(p, scores, sp.sstride, idx, 0, 1, st);
        return e == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
    }
    // the full layer's split parts (if any) use the selection scratch, which is
    // only written after the layer's merge has read them (same stream)
    cudaError_t e = launch_full(p, q, k, v, out, lse, reinterpret_cast<uint8_t*>(ws) + kHeader, ws_bytes - kHeader, st);
    if (e != cudaSuccess) return HS2_ERR_CUDA;
    if (p.topk == 0) return HS2_OK;
    float* scores = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + kHeader);
    const int chunk = sp.chunk > 0 ? sp.chunk : p.nq;
    for (int i0 = 0; i0 < p.nq; i0 += chunk) {
        const int cnt = p.nq - i0 < chunk ? p.nq - i0 : chunk;
        if (sp.tc) {
            e = launch_select_tc(p, q, k, lse, idx, scores, i0, cnt, sp.n_cand_max, st);
            if (e != cudaSuccess) return HS2_ERR_CUDA;
            continue;
        }
        if (sp.sstride > 0) {
            e = launch_score(p, q, k, lse, scores, i0, cnt, sp.sstride, st);
            if (e != cudaSuccess) return HS2_ERR_CUDA;
        }
        e = launch_topk(p, scores, sp.sstride, idx, i0, cnt, st);
        if (e != cudaSuccess) return HS2_ERR_CUDA;
    }
    return HS2_OK;
}

// Block-level selection plan: chunk sums of every candidate tile, over chunks
// of queries whose sums fit kScoreBudget.
struct BlockPlan {
    int64_t n_cand_max = 0;
    int chunk = 0;
    size_t bytes = 0;
};

BlockPlan block_plan(const Problem& p) {
    BlockPlan bp;
    const int64_t cand = p.q_pos0 + p.nq - p.window;  // candidates of the last query
    if (cand <= 0 || p.nq == 0 || p.B == 0 || p.topk == 0) return bp;
    bp.n_cand_max = cand;
    const size_t per_q = block_tc_scratch_bytes(p, 1, cand);
    const int64_t fit = (int64_t)(kScoreBudget / per_q);  // queries whose sums fit the budget
    int64_t chunk = p.nq;
    if (fit < p.nq) {
        // Every CTA of the sweep takes about the same time (it sweeps every
        // candidate tile of its queries) and holds one SM, so a chunk costs whole
        // waves of 148 CTAs: cut the queries into chunks of whole waves.  At 1M
        // that is 4 chunks of 1036 queries (148 CTAs each) instead of 2016, 2016
        // and 64 queries (288, 288 and 12 CTAs: 5 waves).
        const int64_t qt = select_tc_qt(cand, p.hq / p.hkv);
        const int64_t groups = (int64_t)p.hkv * p.B;     // CTAs per qt queries
        const int64_t wave_q = 148 / groups * qt;        // queries of one full wave
        chunk = wave_q > 0 && fit >= wave_q ? fit / wave_q * wave_q : fit / qt * qt;
        if (chunk < qt) chunk = qt;
    }
    bp.chunk = (int)chunk;
    bp.bytes = block_tc_scratch_bytes(p, bp.chunk, cand);
    return bp;
}

size_t block_body_bytes(const Problem& p) {
    const size_t split = full_tc_split_scratch_bytes(p);
    const size_t sel = block_plan(p).bytes;
    return sel > split ? sel : split;
}

bool valid_block(int blk) { return blk == 32 || blk == 64 || blk == 128; }

hs2_status run_block_select(const hs2_shape* shape, int blk, const void* q, const void* k, const void* v, void* out,
                            float* lse, int32_t* idx, void* ws, size_t ws_bytes, hs2_stream_t stream) {
    Problem p;
    hs2_status s = check_shape(shape, &p);
    if (s != HS2_OK) return s;
    if (!valid_block(blk)) return HS2_ERR_UNSUPPORTED;
    if (p.B == 0 || p.nq == 0) return HS2_OK;
    if (!q || !k || !v || !out || !lse || !ws) return HS2_ERR_INVALID_ARG;
    if (p.topk > 0 && !idx) return HS2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
        !aligned(idx, 4) || !aligned(ws, 256))
        return HS2_ERR_INVALID_ARG;
    if (ws_bytes < kHeader + block_body_bytes(p)) return HS2_ERR_WORKSPACE;
    p.err = reinterpret_cast<WsHeader*>(ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* body = reinterpret_cast<uint8_t*>(ws) + kHeader;
    cudaError_t e = launch_full(p, q, k, v, out, lse, body, ws_bytes - kHeader, st);
    if (e != cudaSuccess) return HS2_ERR_CUDA;
    if (p.topk == 0) return HS2_OK;
    const BlockPlan bp = block_plan(p);
    const int chunk = bp.chunk > 0 ? bp.chunk : p.nq;
    for (int i0 = 0; i0 < p.nq; i0 += chunk) {
        const int cnt = p.nq - i0 < chunk ? p.nq - i0 : chunk;
        e = launch_block_select_tc(p, q, k, lse, idx, body, i0, cnt, bp.n_cand_max, blk, st);
        if (e != cudaSuccess) return HS2_ERR_CUDA;
    }
    return HS2_OK;
}

// Context parallelism: a call over one slice of the context's KV cache.  The
// shape describes the slice (kv_len = its rows, q_pos0 = the absolute position
// of query 0) and kv_off is the absolute position of the slice's first key; a
// query may sit before the slice (no key there) or after it (all its keys).
// The kernels see positions shifted by -kv_off.  Prefill-shaped calls only
// (n_q >= 64, the tensor-core paths).
hs2_status check_slice(const hs2_shape* shape, int64_t kv_off, Problem* p) {
    if (shape == nullptr || kv_off < 0) return HS2_ERR_INVALID_ARG;
    if (shape->kv_len < 1 || shape->q_pos0 < 0) return HS2_ERR_INVALID_ARG;
    hs2_shape s = *shape;
    s.q_pos0 = 0;  // the slice rule replaces q_pos0 + n_q <= kv_len
    if (s.kv_len < s.n_q) s.kv_len = s.n_q;
    const hs2_status st = check_shape(&s, p);
    if (st != HS2_OK) return st;
    if (shape->n_q > 0 && shape->n_q < 64) return HS2_ERR_UNSUPPORTED;
    if (shape->q_pos0 + (int64_t)shape->n_q > (int64_t)INT32_MAX + 1) return HS2_ERR_UNSUPPORTED;
    p->kv_len = shape->kv_len;
    p->q_pos0 = shape->q_pos0 - kv_off;
    return HS2_OK;
}

// Selection plan of a slice: candidates of the last query inside the slice.
// The selection runs even when no query has a candidate in the slice (it then
// writes -1 rows and -1 scores), so the plan never has zero candidates.
ScorePlan slice_plan(const Problem& p) {
    ScorePlan sp;
    if (p.nq == 0 || p.B == 0 || p.topk == 0) return sp;
    int64_t cand = p.q_pos0 + p.nq - p.window;  // t_max - window + 1 in slice rows
    if (cand > p.kv_len) cand = p.kv_len;
    if (cand < 1) cand = 1;
    sp.tc = true;
    sp.n_cand_max = cand;
    const size_t per_q = (size_t)p.B * p.hkv * (1024 * 4 + 12);
    int64_t chunk = (int64_t)(kSampleBudget / per_q) / 32 * 32;
    if (chunk < 32) chunk = 32;
    if (chunk > p.nq) chunk = p.nq;
    sp.chunk = (int)chunk;
    sp.bytes = select_tc_scratch_bytes(p, sp.chunk, cand);
    return sp;
}

size_t cp_body_bytes(const Problem& p, int entry) {
    switch (entry) {
        case HS2_ENTRY_CP_ATTN: return full_tc_split_scratch_bytes(p);
        case HS2_ENTRY_CP_SELECT: return slice_plan(p).bytes;
        case HS2_ENTRY_CP_SPARSE: return (size_t)p.B * p.hkv * p.nq * p.topk * 4;
        default: return 0;
    }
}

// Slice calls need a workspace: the error word, then `need` bytes of scratch.
hs2_status check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (ws == nullptr || !aligned(ws, 256)) return HS2_ERR_INVALID_ARG;
    if (ws_bytes < kHeader + need) return HS2_ERR_WORKSPACE;
    return HS2_OK;
}

}  // namespace
}  // namespace hs2

using namespace hs2;

extern "C" {

size_t hs2_workspace_size(const hs2_shape* shape, int entry) {
    Problem p;
    if (check_shape(shape, &p) != HS2_OK) return 0;
    switch (entry) {
        case HS2_ENTRY_SPARSE: return kHeader;
        case HS2_ENTRY_FULL_SELECT:
        case HS2_ENTRY_PREFILL: return kHeader + prefill_body_bytes(p, score_plan(p, false));
        case HS2_ENTRY_BLOCK_SELECT: return kHeader + block_body_bytes(p);
        case HS2_ENTRY_CP_ATTN:
        case HS2_ENTRY_CP_SELECT:
        case HS2_ENTRY_CP_SPARSE: return 0;  // slices: hs2_cp_workspace_size
        case HS2_ENTRY_DECODE: {
            if (p.nq != 1) return 0;
            const ScorePlan sp = score_plan(p, true);
            return kHeader + (sp.bytes + 255) / 256 * 256 + decode_scratch_bytes(p) + topk_chunk_bytes(p, sp.n_cand_max);
        }
        default: return 0;
    }
}

hs2_status hs2_workspace_init(void* ws, size_t ws_bytes, hs2_stream_t stream) {
    if (ws == nullptr || ws_bytes < kHeader || !aligned(ws, 256)) return HS2_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, kHeader, reinterpret_cast<cudaStream_t>(stream)));
}

hs2_status hs2_full_attn_select(const hs2_shape* shape, const void* q, const void* k, const void* v, void* out,
                                float* lse, int32_t* idx, void* ws, size_t ws_bytes, hs2_stream_t stream) {
    return run_full_select(shape, nullptr, false, q, k, v, out, lse, idx, ws, ws_bytes, stream);
}

hs2_status hs2_full_attn_block_select(const hs2_shape* shape, int32_t block, const void* q, const void* k,
                                      const void* v, void* out, float* lse, int32_t* idx, void* ws, size_t ws_bytes,
                                      hs2_stream_t stream) {
    return run_block_select(shape, block, q, k, v, out, lse, idx, ws, ws_bytes, stream);
}

hs2_status hs2_prefill_chunk(const hs2_shape* shape, const void* q, const void* k, const void* v, void* out,
                             float* lse, int32_t* idx, void* ws, size_t ws_bytes, hs2_stream_t stream) {
    return run_full_select(shape, nullptr, false, q, k, v, out, lse, idx, ws, ws_bytes, stream);
}

hs2_status hs2_decode(const hs2_shape* shape, const int64_t* kv_len_per_seq, const void* q, const void* k,
                      const void* v, void* out, float* lse, int32_t* idx, void* ws, size_t ws_bytes,
                      hs2_stream_t stream) {
    if (shape == nullptr) return HS2_ERR_INVALID_ARG;
    hs2_shape s = *shape;
    if (s.n_q != 1 && s.n_q != 0) return HS2_ERR_INVALID_ARG;
    if (s.kv_len < 1 && s.n_q == 1) return HS2_ERR_INVALID_ARG;
    s.q_pos0 = s.kv_len > 0 ? s.kv_len - 1 : 0;  // sequences without a length array end at kv_len - 1
    return run_full_select(&s, kv_len_per_seq, true, q, k, v, out, lse, idx, ws, ws_bytes, stream);
}

namespace hs2 {
namespace {
hs2_status run_sparse(const hs2_shape* shape, const int64_t* seq_len, const void* q, const void* k, const void* v,
                      const int32_t* idx, void* out, void* ws, size_t ws_bytes, hs2_stream_t stream) {
    Problem p;
    hs2_status s = check_shape(shape, &p);
    if (s != HS2_OK) return s;
    if (seq_len && !aligned(seq_len, 8)) return HS2_ERR_INVALID_ARG;
    p.seq_len = seq_len;
    if (p.B == 0 || p.nq == 0) return HS2_OK;
    if (!q || !k || !v || !out || (p.topk > 0 && !idx)) return HS2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(idx, 4))
        return HS2_ERR_INVALID_ARG;
    if (ws != nullptr) {
        if (ws_bytes < kHeader || !aligned(ws, 256)) return HS2_ERR_WORKSPACE;
        p.err = reinterpret_cast<WsHeader*>(ws);
    } else if (ws_bytes != 0) {
        return HS2_ERR_INVALID_ARG;
    }
    return cuda_status(launch_sparse(p, q, k, v, idx, out, reinterpret_cast<cudaStream_t>(stream)));
}
}  // namespace
}  // namespace hs2

hs2_status hs2_kv_bridge(const hs2_bridge_shape* s, const int64_t* seq_pos, const void* hidden, const void* w_kv,
                         void* k_cache, void* v_cache, void* ws, size_t ws_bytes, hs2_stream_t stream) {
    if (s == nullptr) return HS2_ERR_INVALID_ARG;
    if (s->reserved != 0 || s->batch < 0 || s->n_new < 0 || s->d_model <= 0 || s->h_kv <= 0 || s->kv_cap <= 0 ||
        s->pos0 < 0)
        return HS2_ERR_INVALID_ARG;
    if (s->d_model % 64 != 0 || (s->head_dim != 64 && s->head_dim != 128) || (s->h_kv * s->head_dim) % 256 != 0 ||
        s->h_kv > 64)
        return HS2_ERR_UNSUPPORTED;
    const int64_t n_rows = (int64_t)s->batch * s->n_new;
    if ((n_rows + 127) / 128 > 65535) return HS2_ERR_UNSUPPORTED;  // token tiles in one grid dimension
    if (seq_pos == nullptr && s->pos0 + s->n_new > s->kv_cap) return HS2_ERR_INVALID_ARG;
    if (n_rows == 0) return HS2_OK;
    if (!hidden || !w_kv || !k_cache || !v_cache) return HS2_ERR_INVALID_ARG;
    if (!aligned(hidden, 16) || !aligned(w_kv, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        (seq_pos && !aligned(seq_pos, 8)))
        return HS2_ERR_INVALID_ARG;
    if (ws != nullptr && (ws_bytes < kHeader || !aligned(ws, 256))) return HS2_ERR_WORKSPACE;
    if (ws == nullptr && ws_bytes != 0) return HS2_ERR_INVALID_ARG;
    WsHeader* err = ws ? reinterpret_cast<WsHeader*>(ws) : nullptr;
    // a workspace large enough for the split partials enables the split path
    const size_t split = bridge_split_bytes(n_rows, s->d_model, s->h_kv, s->head_dim);
    float* part = (ws != nullptr && split > 0 && ws_bytes >= kHeader + split)
                      ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + kHeader)
                      : nullptr;
    return cuda_status(launch_bridge(n_rows, s->n_new, s->d_model, s->h_kv, s->head_dim, s->pos0, s->kv_cap, seq_pos,
                                     hidden, w_kv, k_cache, v_cache, err, reinterpret_cast<cudaStream_t>(stream), part));
}

size_t hs2_kv_bridge_workspace_size(const hs2_bridge_shape* s) {
    if (s == nullptr || s->batch < 0 || s->n_new < 0 || s->d_model <= 0 || s->d_model % 64 != 0 || s->h_kv <= 0 ||
        (s->head_dim != 64 && s->head_dim != 128))
        return 0;
    return kHeader + bridge_split_bytes((int64_t)s->batch * s->n_new, s->d_model, s->h_kv, s->head_dim);
}

hs2_status hs2_sparse_attn(const hs2_shape* shape, const void* q, const void* k, const void* v, const int32_t* idx,
                           void* out, void* ws, size_t ws_bytes, hs2_stream_t stream) {
    return run_sparse(shape, nullptr, q, k, v, idx, out, ws, ws_bytes, stream);
}

hs2_status hs2_decode_sparse(const hs2_shape* shape, const int64_t* kv_len_per_seq, const void* q, const void* k,
                             const void* v, const int32_t* idx, void* out, void* ws, size_t ws_bytes,
                             hs2_stream_t stream) {
    if (shape == nullptr) return HS2_ERR_INVALID_ARG;
    hs2_shape s = *shape;
    if (s.n_q != 1 && s.n_q != 0) return HS2_ERR_INVALID_ARG;
    if (s.kv_len < 1 && s.n_q == 1) return HS2_ERR_INVALID_ARG;
    s.q_pos0 = s.kv_len > 0 ? s.kv_len - 1 : 0;
    return run_sparse(&s, kv_len_per_seq, q, k, v, idx, out, ws, ws_bytes, stream);
}

hs2_status hs2_swa_branches(const hs2_shape* shape, const void* q, const void* k_swa, const void* v_swa,
                            const void* k, const void* v, const int32_t* idx, void* out_swa, float* lse_swa,
                            void* out_sel, float* lse_sel, void* ws, size_t ws_bytes, hs2_stream_t stream) {
    Problem p;
    hs2_status s = check_shape(shape, &p);
    if (s != HS2_OK) return s;
    if (p.B == 0 || p.nq == 0) return HS2_OK;
    if (!q || !k_swa || !v_swa || !k || !v || !out_swa || !lse_swa || !out_sel || !lse_sel ||
        (p.topk > 0 && !idx))
        return HS2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_swa, 16) || !aligned(v_swa, 16) || !aligned(k, 16) || !aligned(v, 16) ||
        !aligned(idx, 4) || !aligned(out_swa, 16) || !aligned(out_sel, 16) || !aligned(lse_swa, 4) ||
        !aligned(lse_sel, 4))
        return HS2_ERR_INVALID_ARG;
    if (ws != nullptr) {
        if (ws_bytes < kHeader || !aligned(ws, 256)) return HS2_ERR_WORKSPACE;
        p.err = reinterpret_cast<WsHeader*>(ws);
    } else if (ws_bytes != 0) {
        return HS2_ERR_INVALID_ARG;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // selected branch: the selected rows of the shared cache alone
    cudaError_t e = launch_sparse(p, q, k, v, idx, out_sel, st, 0, lse_sel);
    if (e != cudaSuccess) return HS2_ERR_CUDA;
    // window branch: the same kernel with no selection, over the branch's own cache
    Problem pw = p;
    pw.topk = 0;
    return cuda_status(launch_sparse(pw, q, k_swa, v_swa, nullptr, out_swa, st, 1, lse_swa));
}

size_t hs2_cp_workspace_size(const hs2_shape* shape, int64_t kv_off, int entry) {
    Problem p;
    if (check_slice(shape, kv_off, &p) != HS2_OK) return 0;
    if (entry != HS2_ENTRY_CP_ATTN && entry != HS2_ENTRY_CP_SELECT && entry != HS2_ENTRY_CP_SPARSE) return 0;
    return kHeader + cp_body_bytes(p, entry);
}

hs2_status hs2_cp_attn_partial(const hs2_shape* shape, int64_t kv_off, const void* q, const void* k, const void* v,
                               void* out, float* lse, void* ws, size_t ws_bytes, hs2_stream_t stream) {
    Problem p;
    hs2_status s = check_slice(shape, kv_off, &p);
    if (s != HS2_OK) return s;
    if (p.B == 0 || p.nq == 0) return HS2_OK;
    if (!q || !k || !v || !out || !lse) return HS2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4))
        return HS2_ERR_INVALID_ARG;
    if ((s = check_ws(ws, ws_bytes, cp_body_bytes(p, HS2_ENTRY_CP_ATTN))) != HS2_OK) return s;
    p.err = reinterpret_cast<WsHeader*>(ws);
    return cuda_status(launch_full_tc(p, q, k, v, out, lse, reinterpret_cast<uint8_t*>(ws) + kHeader,
                                      ws_bytes - kHeader, reinterpret_cast<cudaStream_t>(stream)));
}

hs2_status hs2_cp_select_local(const hs2_shape* shape, int64_t kv_off, const void* q, const void* k,
                               const float* lse, int32_t* idx, float* score, void* ws, size_t ws_bytes,
                               hs2_stream_t stream) {
    Problem p;
    hs2_status s = check_slice(shape, kv_off, &p);
    if (s != HS2_OK) return s;
    if (p.B == 0 || p.nq == 0 || p.topk == 0) return HS2_OK;
    if (!q || !k || !lse || !idx || !score) return HS2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(lse, 4) || !aligned(idx, 4) || !aligned(score, 4))
        return HS2_ERR_INVALID_ARG;
    const ScorePlan sp = slice_plan(p);
    if ((s = check_ws(ws, ws_bytes, sp.bytes)) != HS2_OK) return s;
    p.err = reinterpret_cast<WsHeader*>(ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void* scratch = reinterpret_cast<uint8_t*>(ws) + kHeader;
    const int chunk = sp.chunk > 0 ? sp.chunk : p.nq;
    for (int i0 = 0; i0 < p.nq; i0 += chunk) {
        const int cnt = p.nq - i0 < chunk ? p.nq - i0 : chunk;
        const cudaError_t e = launch_select_tc(p, q, k, lse, idx, scratch, i0, cnt, sp.n_cand_max, st, score);
        if (e != cudaSuccess) return HS2_ERR_CUDA;
    }
    return HS2_OK;
}

hs2_status hs2_cp_sparse_partial(const hs2_shape* shape, int64_t kv_off, const void* q, const void* k,
                                 const void* v, const int32_t* idx, void* out, float* lse, void* ws, size_t ws_bytes,
                                 hs2_stream_t stream) {
    Problem p;
    hs2_status s = check_slice(shape, kv_off, &p);
    if (s != HS2_OK) return s;
    if (p.B == 0 || p.nq == 0) return HS2_OK;
    if (!q || !k || !v || !out || !lse || (p.topk > 0 && !idx)) return HS2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
        !aligned(idx, 4))
        return HS2_ERR_INVALID_ARG;
    if ((s = check_ws(ws, ws_bytes, cp_body_bytes(p, HS2_ENTRY_CP_SPARSE))) != HS2_OK) return s;
    p.err = reinterpret_cast<WsHeader*>(ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t* local = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(ws) + kHeader);
    const int64_t rows = (int64_t)p.B * p.hkv * p.nq;
    cudaError_t e = launch_cp_idx_local(rows, p.topk, idx, kv_off, p.kv_len, local, st);
    if (e != cudaSuccess) return HS2_ERR_CUDA;
    return cuda_status(launch_sparse(p, q, k, v, p.topk > 0 ? local : nullptr, out, st, 1, lse));
}

hs2_status hs2_cp_combine(int32_t n_parts, int64_t n_rows, int32_t head_dim, const void* out_parts,
                          const float* lse_parts, void* out, float* lse, hs2_stream_t stream) {
    if (n_parts < 1 || n_rows < 0) return HS2_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return HS2_ERR_UNSUPPORTED;
    if (n_rows == 0) return HS2_OK;
    if (!out_parts || !lse_parts || !out || !lse) return HS2_ERR_INVALID_ARG;
    if (!aligned(out_parts, 16) || !aligned(out, 16) || !aligned(lse_parts, 4) || !aligned(lse, 4))
        return HS2_ERR_INVALID_ARG;
    return cuda_status(launch_cp_combine(n_parts, n_rows, head_dim, out_parts, lse_parts, out, lse,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

hs2_status hs2_cp_select_merge(const hs2_shape* shape, int32_t n_parts, const int64_t* kv_offs,
                               const int32_t* idx_parts, const float* score_parts, int32_t* idx,
                               hs2_stream_t stream) {
    Problem p;
    hs2_status s = check_shape(shape, &p);
    if (s != HS2_OK) return s;
    if (n_parts < 1 || kv_offs == nullptr) return HS2_ERR_INVALID_ARG;
    if (n_parts > cp_max_parts()) return HS2_ERR_UNSUPPORTED;
    for (int i = 0; i < n_parts; ++i)
        if (kv_offs[i] < 0 || (i > 0 && kv_offs[i] <= kv_offs[i - 1])) return HS2_ERR_INVALID_ARG;
    if (p.B == 0 || p.nq == 0 || p.topk == 0) return HS2_OK;
    if (!idx_parts || !score_parts || !idx) return HS2_ERR_INVALID_ARG;
    if (!aligned(idx_parts, 4) || !aligned(score_parts, 4) || !aligned(idx, 4)) return HS2_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)p.B * p.hkv * p.nq;
    return cuda_status(launch_cp_select_merge(n_parts, rows, p.topk, idx_parts, score_parts, kv_offs, idx,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

hs2_status hs2_get_device_status(void* ws, hs2_stream_t stream, uint32_t* info) {
    if (ws == nullptr || !aligned(ws, 256)) return HS2_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t h[4] = {0, 0, 0, 0};
    if (cudaStreamSynchronize(st) != cudaSuccess) return HS2_ERR_CUDA;
    if (cudaMemcpy(h, ws, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return HS2_ERR_CUDA;
    if (h[0] != 0) {
        if (cudaMemset(ws, 0, sizeof h) != cudaSuccess) return HS2_ERR_CUDA;
    }
    if (info) {
        for (int u = 0; u < 4; ++u) info[u] = h[u];
    }
    if (h[0] == HS2_ERR_DEVICE_CHECK) return HS2_ERR_DEVICE_CHECK;
    if (h[0] == HS2_ERR_TIMEOUT) return HS2_ERR_TIMEOUT;
    return h[0] == 0 ? HS2_OK : HS2_ERR_DEVICE_CHECK;
}

hs2_status hs2_select_retry_rows(const hs2_shape* shape, const void* ws, size_t ws_bytes, hs2_stream_t stream,
                                 int64_t* n_rows) {
    Problem p;
    hs2_status s = check_shape(shape, &p);
    if (s != HS2_OK) return s;
    if (n_rows == nullptr || ws == nullptr || !aligned(ws, 256)) return HS2_ERR_INVALID_ARG;
    *n_rows = 0;
    const ScorePlan sp = score_plan(p, false);
    if (!sp.tc || p.topk == 0 || p.B == 0 || p.nq == 0) return HS2_OK;  // no sampled selection pass ran
    if (ws_bytes < kHeader + prefill_body_bytes(p, sp)) return HS2_ERR_WORKSPACE;
    const int i_last = (p.nq - 1) / sp.chunk * sp.chunk;  // first query of the last chunk
    const int cnt = p.nq - i_last;
    const size_t rows = (size_t)p.B * p.hkv * cnt;
    const size_t off = kHeader + select_tc_status_offset(p, cnt, sp.n_cand_max);
    std::vector<int32_t> mark(rows);
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return HS2_ERR_CUDA;
    if (cudaMemcpy(mark.data(), reinterpret_cast<const uint8_t*>(ws) + off, rows * sizeof(int32_t),
                   cudaMemcpyDeviceToHost) != cudaSuccess)
        return HS2_ERR_CUDA;
    int64_t n = 0;
    for (int32_t m : mark) n += m != 0;
    *n_rows = n;
    return HS2_OK;
}

const char* hs2_status_string(hs2_status status) {
    switch (status) {
        case HS2_OK: return "ok";
        case HS2_ERR_INVALID_ARG: return "invalid argument";
        case HS2_ERR_UNSUPPORTED: return "unsupported shape";
        case HS2_ERR_WORKSPACE: return "workspace too small";
        case HS2_ERR_CUDA: return "CUDA error";
        case HS2_ERR_DEVICE_CHECK: return "device-side input check failed";
        case HS2_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

uint64_t hs2_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

hs2_status hs2_profile_start(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (auto& r : g_prof_recs) {
        g_prof_pool.push_back(r.a);
        g_prof_pool.push_back(r.b);
    }
    g_prof_recs.clear();
    g_prof_on.store(true);
    return HS2_OK;
}

hs2_status hs2_profile_stop(uint32_t n_kinds, float* total_ms, uint64_t* launches) {
    g_prof_on.store(false);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (uint32_t u = 0; u < n_kinds; ++u) {
        if (total_ms) total_ms[u] = 0.f;
        if (launches) launches[u] = 0;
    }
    hs2_status st = HS2_OK;
    for (auto& r : g_prof_recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            st = HS2_ERR_CUDA;
        if (r.kid < n_kinds) {
            if (total_ms) total_ms[r.kid] += ms;
            if (launches) launches[r.kid] += 1;
        }
        g_prof_pool.push_back(r.a);
        g_prof_pool.push_back(r.b);
    }
    g_prof_recs.clear();
    return st;
}

int hs2_is_checked_build(void) {
#ifdef HS2_CHECKED
    return 1;
#else
    return 0;
#endif
}

}  // extern "C"
