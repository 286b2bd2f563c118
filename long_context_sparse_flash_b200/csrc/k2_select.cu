// k2_select.cu -- K2: token-level selection of HySparse2 (xiawanshe.com report,
// section "Token级选择": per-token choice of 1024 older tokens beside the forced
// 128-token window; davidyin.dev notes, "HySparse2 的解法": no trained indexer,
// so the score comes from the full-attention layer itself).
//
// Score of candidate j for KV group g at query t:
//     score = sum_{h in g} 2^(s2_{h,j} - lse2_h),  s2 = scale*log2(e)*<q_h,k_j>,
// recomputed from the LSE that K1 wrote.  Part 1 (k2_score_kernel) computes the
// scores with mma.sync in the transposed form S^T = K Q^T, so one 16-key x
// 8-column tile holds one query's 8 heads (G = 8) in one row of the fragment and
// the group sum is two in-thread adds plus two quad shuffles.  Part 2
// (k2_topk_kernel) selects the top-k of each (query, group) row exactly: a
// 3-pass (11, 11, 10 bits) radix select on the fp32 bit patterns (non-negative
// floats order like their bits; histogram updates aggregated per warp with
// match_any) finds the k-th key, then one ordered pass keeps every key above
// it plus the lowest-index keys equal to it, writing indices ascending.
#include "hs2_kernels.h"

namespace hs2 {

namespace {

constexpr int SC_WARPS = 8;
constexpr int SC_BN = 64;  // keys per staged tile

template <int D, int G>
__global__ void __launch_bounds__(SC_WARPS * 32) k2_score_kernel(Problem p, const __nv_bfloat16* __restrict__ q,
                                                                  const __nv_bfloat16* __restrict__ k,
                                                                  const float* __restrict__ lse,
                                                                  float* __restrict__ scores, int i_begin,
                                                                  int i_count, int64_t sstride,
                                                                  int64_t keys_per_split, int splits) {
    constexpr int CH = D / 8;
    constexpr int QPN = 8 / G;                   // queries per 8-column n-tile
    constexpr int QPC = SC_WARPS * 2 * QPN;      // queries per CTA
    constexpr int T_BYTES = SC_BN * D * 2;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.y;
    const int b = blockIdx.z / splits, split = blockIdx.z % splits;
    const int64_t pos0 = seq_pos0(p, b, KID_SCORE);
    const int qc0 = blockIdx.x * QPC;            // first query of the CTA, relative to i_begin
    const int q_end = min(qc0 + QPC, i_count);   // exclusive
    if (qc0 >= q_end) return;
    const int64_t t_hi = pos0 + i_begin + q_end - 1;
    const int64_t cand_end = t_hi - p.window + 1;  // candidates are j < cand_end
    const int64_t j_lo = (int64_t)split * keys_per_split;
    const int64_t j_hi = min(j_lo + keys_per_split, cand_end);
    if (j_lo >= j_hi) return;
    const int n_tiles = (int)((j_hi - j_lo + SC_BN - 1) / SC_BN);

    const __nv_bfloat16* kg = k + ((int64_t)(b * p.hkv + g) * p.kv_len) * D;
    const uint32_t s_t = smem_u32(smem);
    auto load_tile = [&](int kt, int stage) {
        const uint32_t sk = s_t + stage * T_BYTES;
        for (int c = tid; c < SC_BN * CH; c += SC_WARPS * 32) {
            const int r = c / CH, ch = c % CH;
            const int64_t j = j_lo + (int64_t)kt * SC_BN + r;
            const bool ok = j < j_hi;
            cp_async16(sk + swz<CH>(r, ch), kg + (ok ? j : 0) * D + ch * 8, ok ? 16 : 0);
        }
    };
    load_tile(0, 0);
    cp_async_commit();

    // B fragments (Q^T) of this warp's two n-tiles: column c = query (c / G), head (c % G)
    uint32_t qb[2][D / 16][2];
    float l2[2][2];          // lse * log2(e) of this thread's two columns per n-tile
    int64_t t_col[2][2];     // absolute position of the column's query (-1: none)
    int row_col[2][2];       // score row of the column's query
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        {
            const int c = lane >> 2;  // column this thread feeds to the B fragment
            const int qi = qc0 + (warp * 2 + nt) * QPN + c / G;
            const int hh = c % G;
            const bool ok = qi < q_end;
            const int i = i_begin + (ok ? qi : qc0);
            const __nv_bfloat16* qrow = q + ((int64_t)(b * p.hq + g * G + hh) * p.nq + i) * D;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int d0 = ks * 16 + 2 * (lane & 3);
                qb[nt][ks][0] = ok ? *reinterpret_cast<const uint32_t*>(qrow + d0) : 0u;
                qb[nt][ks][1] = ok ? *reinterpret_cast<const uint32_t*>(qrow + d0 + 8) : 0u;
            }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int c = 2 * (lane & 3) + e;  // column of accumulator element e
            const int qi = qc0 + (warp * 2 + nt) * QPN + c / G;
            const int hh = c % G;
            const bool ok = qi < q_end;
            const int i = i_begin + (ok ? qi : qc0);
            l2[nt][e] = ok ? lse[(int64_t)(b * p.hq + g * G + hh) * p.nq + i] * kLog2e : INFINITY;
            t_col[nt][e] = ok ? pos0 + i : -1;
            row_col[nt][e] = qi;
        }
    }

    for (int kt = 0; kt < n_tiles; ++kt) {
        if (kt + 1 < n_tiles) {
            load_tile(kt + 1, (kt + 1) & 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint32_t sk = s_t + (kt & 1) * T_BYTES;
        const int64_t j_tile = j_lo + (int64_t)kt * SC_BN;
#pragma unroll
        for (int mt = 0; mt < SC_BN / 16; ++mt) {
            float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t a[4];
                const int mi = lane >> 3;
                ldsm_x4(a, sk + swz<CH>(mt * 16 + (mi & 1) * 8 + (lane & 7), 2 * ks + (mi >> 1)));
                mma16816(c[0], a, qb[0][ks]);
                mma16816(c[1], a, qb[1][ks]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                float pe[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) pe[e] = ex2(c[nt][e] * p.scale_log2 - l2[nt][e & 1]);
#pragma unroll
                for (int r = 0; r < 2; ++r) {  // key rows lane/4 and lane/4 + 8
                    const int64_t j = j_tile + mt * 16 + (lane >> 2) + 8 * r;
                    float v0 = pe[2 * r], v1 = pe[2 * r + 1];
                    if (G == 8) {
                        float sum = v0 + v1;
                        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                        if ((lane & 3) == 0 && j <= t_col[nt][0] - p.window && j < j_hi)
                            scores[((int64_t)(b * p.hkv + g) * i_count + row_col[nt][0]) * sstride + j] = sum;
                    } else if (G == 4) {
                        float sum = v0 + v1;
                        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                        if ((lane & 1) == 0 && j <= t_col[nt][0] - p.window && j < j_hi)
                            scores[((int64_t)(b * p.hkv + g) * i_count + row_col[nt][0]) * sstride + j] = sum;
                    } else if (G == 2) {
                        const float sum = v0 + v1;
                        if (j <= t_col[nt][0] - p.window && j < j_hi)
                            scores[((int64_t)(b * p.hkv + g) * i_count + row_col[nt][0]) * sstride + j] = sum;
                    } else {
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const float val = e ? v1 : v0;
                            if (j <= t_col[nt][e] - p.window && j < j_hi)
                                scores[((int64_t)(b * p.hkv + g) * i_count + row_col[nt][e]) * sstride + j] = val;
                        }
                    }
                }
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------

constexpr int TK_THREADS = 1024;
constexpr int TK_WARPS = TK_THREADS / 32;
constexpr int TK_BINS = 2048;
constexpr int TK_SAMPLES = 8192;  // keys sampled per row for the threshold
constexpr int TK_CAP = 8192;      // survivor buffer (keys and indices in shared memory)
constexpr int TK_DYN_SMEM = 2 * TK_CAP * 4;

struct TopkSmem {
    uint32_t hist[TK_BINS];
    uint32_t warp_tot[TK_WARPS];
    uint32_t warp_tot2[TK_WARPS];
    uint32_t digit, k_rem;
};

// exclusive prefix of per-thread counts over the block; returns the prefix,
// writes the block total
__device__ __forceinline__ uint32_t block_excl_sum(uint32_t x, uint32_t* warp_tot, uint32_t& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < TK_WARPS; ++w) {
        const uint32_t v = warp_tot[w];
        before += (w < warp) ? v : 0u;
        tot += v;
    }
    total = tot;
    return before + incl - x;
}

// Radix digit boundaries: bits [31,21], [20,10], [9,0] of the fp32 score.
__device__ __forceinline__ void digit_of(int pass, int& shift, uint32_t& mask) {
    shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    mask = pass == 2 ? 1023u : 2047u;
}

// Exact top-k of one row over all n keys in global memory (the fallback):
// 3-pass radix select for the k-th key, then an ordered pass, indices ascending.
__device__ void topk_exact_global(const uint32_t* __restrict__ key, int n, int topk, int32_t* __restrict__ orow,
                                  TopkSmem& sm, float* __restrict__ srow = nullptr) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int n4 = n / 4;  // rows start 16-byte aligned (sstride is a multiple of 4)
    // radix select: the key value of the topk-th largest (non-negative floats
    // order like their bit patterns), three passes of 11, 11 and 10 bits
    uint32_t prefix = 0, pmask = 0;
    uint32_t k_rem = (uint32_t)topk;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        int shift;
        uint32_t dmask;
        digit_of(pass, shift, dmask);
        for (int u = tid; u < TK_BINS; u += TK_THREADS) sm.hist[u] = 0;
        __syncthreads();
        auto add = [&](uint32_t x, bool valid) {
            const bool part = valid && (x & pmask) == prefix;
            const uint32_t act = __ballot_sync(0xffffffffu, part);
            if (part) {
                const uint32_t bin = (x >> shift) & dmask;
                const uint32_t peers = __match_any_sync(act, bin);
                if (lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bin], (uint32_t)__popc(peers));
            }
        };
        for (int base = 0; base < n4; base += TK_THREADS) {
            const int j4 = base + tid;
            uint4 x = make_uint4(0u, 0u, 0u, 0u);
            if (j4 < n4) x = reinterpret_cast<const uint4*>(key)[j4];
            const bool ok = j4 < n4;
            add(x.x, ok);
            add(x.y, ok);
            add(x.z, ok);
            add(x.w, ok);
        }
        {  // tail of up to 3 keys; every lane takes part in the warp-wide vote
            const int j = n4 * 4 + tid;
            const bool ok = tid < 32 && j < n;
            if (tid < 32) add(ok ? key[j] : 0u, ok);
        }
        __syncthreads();
        if (tid < 32) {
            // lane l owns bins [64*(31-l), 64*(31-l)+63], so lane order is descending digit
            uint32_t s = 0;
            const int nb = (int)dmask + 1;
            const int per = nb / 32;
            for (int u = 0; u < per; ++u) s += sm.hist[per * (31 - lane) + u];
            uint32_t incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const uint32_t excl = incl - s;
            if (excl < k_rem && k_rem <= incl) {
                uint32_t above = excl;
                for (int u = per - 1; u >= 0; --u) {
                    const uint32_t c = sm.hist[per * (31 - lane) + u];
                    if (above + c >= k_rem) {
                        sm.digit = (uint32_t)(per * (31 - lane) + u);
                        sm.k_rem = k_rem - above;
                        break;
                    }
                    above += c;
                }
            }
        }
        __syncthreads();
        prefix |= sm.digit << shift;
        pmask |= dmask << shift;
        k_rem = sm.k_rem;
        __syncthreads();
    }
    const uint32_t kth = prefix;
    const uint32_t need_eq = k_rem;  // how many keys equal to kth are taken (lowest j first)

    // ordered pass: keep keys > kth and the first need_eq keys == kth, ascending j;
    // each thread takes 4 consecutive keys per step
    uint32_t eq_seen = 0, written = 0;
    for (int base = 0; base < n; base += 4 * TK_THREADS) {
        const int j0 = base + 4 * tid;
        uint32_t x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) x[u] = (j0 + u < n) ? key[j0 + u] : 0u;
        uint32_t neq = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) neq += (j0 + u < n && x[u] == kth) ? 1u : 0u;
        uint32_t eq_tot;
        uint32_t eq_rank = eq_seen + block_excl_sum(neq, sm.warp_tot, eq_tot);
        bool take[4];
        uint32_t ntake = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const bool valid = j0 + u < n;
            const bool eq = valid && x[u] == kth;
            take[u] = (valid && x[u] > kth) || (eq && eq_rank < need_eq);
            eq_rank += eq ? 1u : 0u;
            ntake += take[u] ? 1u : 0u;
        }
        __syncthreads();
        uint32_t take_tot;
        uint32_t pos = written + block_excl_sum(ntake, sm.warp_tot2, take_tot);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (take[u]) {
                if (srow) srow[pos] = __uint_as_float(x[u]);
                orow[pos++] = j0 + u;
            }
        eq_seen += eq_tot;
        written += take_tot;
        __syncthreads();
    }
}


// Exact radix select over n keys (fp32 bit patterns) of a shared-memory array:
// the K-th largest key value and how many keys equal to it belong to the top K.
__device__ void block_kth_shared(const uint32_t* keys, int n, uint32_t K, TopkSmem& sm, uint32_t& kth,
                                 uint32_t& need_eq) {
    const int tid = threadIdx.x, lane = tid & 31;
    uint32_t prefix = 0, pmask = 0, k_rem = K;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        int shift;
        uint32_t dmask;
        digit_of(pass, shift, dmask);
        for (int u = tid; u < TK_BINS; u += TK_THREADS) sm.hist[u] = 0;
        __syncthreads();
        for (int base = 0; base < n; base += TK_THREADS) {
            const int j = base + tid;
            const bool valid = j < n;
            const uint32_t x = valid ? keys[j] : 0u;
            const bool part = valid && (x & pmask) == prefix;
            const uint32_t act = __ballot_sync(0xffffffffu, part);
            if (part) {
                const uint32_t bin = (x >> shift) & dmask;
                const uint32_t peers = __match_any_sync(act, bin);
                if (lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bin], (uint32_t)__popc(peers));
            }
        }
        __syncthreads();
        if (tid < 32) {
            uint32_t s = 0;
            const int per = ((int)dmask + 1) / 32;
            for (int u = 0; u < per; ++u) s += sm.hist[per * (31 - lane) + u];
            uint32_t incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const uint32_t excl = incl - s;
            if (excl < k_rem && k_rem <= incl) {
                uint32_t above = excl;
                for (int u = per - 1; u >= 0; --u) {
                    const uint32_t c = sm.hist[per * (31 - lane) + u];
                    if (above + c >= k_rem) {
                        sm.digit = (uint32_t)(per * (31 - lane) + u);
                        sm.k_rem = k_rem - above;
                        break;
                    }
                    above += c;
                }
            }
        }
        __syncthreads();
        prefix |= sm.digit << shift;
        pmask |= dmask << shift;
        k_rem = sm.k_rem;
        __syncthreads();
    }
    kth = prefix;
    need_eq = k_rem;
}

// Exact top K of the n (key, index) pairs in shared memory, which are in index
// order: the K-th key, then one ordered pass that writes the indices of the keys
// above it and of the first keys equal to it, ascending, to orow.
__device__ void block_topk_ordered(const uint32_t* lk, const uint32_t* lj, int n, int topk, int32_t* orow,
                                   TopkSmem& sm) {
    const int tid = threadIdx.x;
    uint32_t kth, need_eq;
    block_kth_shared(lk, n, (uint32_t)topk, sm, kth, need_eq);
    uint32_t eq_seen = 0, written = 0;
    for (int base = 0; base < n; base += 4 * TK_THREADS) {
        const int e0 = base + 4 * tid;
        uint32_t x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) x[u] = (e0 + u < n) ? lk[e0 + u] : 0u;
        uint32_t neq = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) neq += (e0 + u < n && x[u] == kth) ? 1u : 0u;
        uint32_t eq_tot;
        uint32_t eq_rank = eq_seen + block_excl_sum(neq, sm.warp_tot, eq_tot);
        bool take[4];
        uint32_t ntake = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const bool valid = e0 + u < n;
            const bool eq = valid && x[u] == kth;
            take[u] = (valid && x[u] > kth) || (eq && eq_rank < need_eq);
            eq_rank += eq ? 1u : 0u;
            ntake += take[u] ? 1u : 0u;
        }
        __syncthreads();
        uint32_t take_tot;
        uint32_t pos = written + block_excl_sum(ntake, sm.warp_tot2, take_tot);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (take[u]) orow[pos++] = (int32_t)lj[e0 + u];
        eq_seen += eq_tot;
        written += take_tot;
        __syncthreads();
    }
}

// One row per CTA.  Fast path: a threshold tau from 8192 keys sampled at a
// fixed stride (the r-th largest, r = L + 4.5 sqrt(L) + 2 with L = K s / n the
// expected number of samples above the K-th best key; tau = 0 when n fits the
// survivor buffer), one streaming pass that compacts the keys >= tau, in j
// order, into shared memory, then the exact select over those survivors.  A
// row with fewer than K survivors (tau too high) or more than the buffer holds
// (e.g. many equal scores) takes the exact passes over the whole row instead.
//
// Chunk mode (chunk_len > 0, one query per sequence): blockIdx.x is a chunk of
// chunk_len candidates of the row; the CTA writes the chunk's exact top-min(K, n)
// as LOCAL indices, ascending, with their scores, to cidx / cscore [row][chunk][K]
// (-1 padded), and k2_chunk_merge_kernel gives the row's top K.
__global__ void __launch_bounds__(TK_THREADS) k2_topk_kernel(Problem p, const float* __restrict__ scores,
                                                             int64_t sstride, int32_t* __restrict__ idx,
                                                             int i_begin, int i_count, int64_t chunk_len,
                                                             int32_t* __restrict__ cidx, float* __restrict__ cscore) {
    __shared__ TopkSmem sm;
    extern __shared__ __align__(16) uint32_t tk_dyn[];
    uint32_t* lk = tk_dyn;            // survivor keys (also the samples, before the compaction)
    uint32_t* lj = tk_dyn + TK_CAP;   // survivor indices
    const int tid = threadIdx.x;
    const bool chunked = chunk_len > 0;
    const int qi = chunked ? 0 : blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int i = i_begin + qi;
    const int64_t pos0 = seq_pos0(p, b, KID_TOPK);
    const int64_t t = pos0 + i;
    const int64_t n64 = t - p.window + 1;
    const int64_t c0 = chunked ? (int64_t)blockIdx.x * chunk_len : 0;  // first candidate of the chunk
    int64_t n_here = n64 - c0;
    if (chunked && n_here > chunk_len) n_here = chunk_len;
    const int n = n_here > 0 ? (int)n_here : 0;
    const int64_t row = (int64_t)(b * p.hkv + g);
    int32_t* orow = chunked ? cidx + (row * gridDim.x + blockIdx.x) * p.topk : idx + (row * p.nq + i) * p.topk;
    float* srow = chunked ? cscore + (row * gridDim.x + blockIdx.x) * p.topk : nullptr;
    const uint32_t* key = reinterpret_cast<const uint32_t*>(scores + (row * i_count + qi) * sstride + c0);
    if (n <= p.topk) {
        for (int r = tid; r < p.topk; r += TK_THREADS) {
            orow[r] = r < n ? r : -1;
            if (srow) srow[r] = r < n ? __uint_as_float(key[r]) : -1.f;
        }
        return;
    }

    // threshold
    uint32_t tau = 0u;
    if (n > TK_CAP) {
        const int stride = n / TK_SAMPLES;  // >= 1
        for (int u = tid; u < TK_SAMPLES; u += TK_THREADS) lk[u] = key[(int64_t)u * stride];
        __syncthreads();
        const float lam = (float)p.topk * (float)TK_SAMPLES / (float)n;
        const int r = (int)ceilf(lam + 4.5f * sqrtf(lam) + 2.f);
        if (r < TK_SAMPLES) {
            uint32_t need_eq;
            block_kth_shared(lk, TK_SAMPLES, (uint32_t)r, sm, tau, need_eq);
        }
        __syncthreads();  // samples consumed before the compaction overwrites them
    }

    // ordered compaction of the keys >= tau: 16 consecutive keys per thread per
    // step, their four 16-byte loads issued together
    constexpr int KPT = 16;
    uint32_t cnt = 0;
    for (int base = 0; base < n; base += KPT * TK_THREADS) {
        const int j0 = base + KPT * tid;
        uint32_t x[KPT];
        if (j0 + KPT - 1 < n) {
#pragma unroll
            for (int v = 0; v < KPT / 4; ++v) {
                const uint4 v4 = *reinterpret_cast<const uint4*>(key + j0 + 4 * v);
                x[4 * v] = v4.x, x[4 * v + 1] = v4.y, x[4 * v + 2] = v4.z, x[4 * v + 3] = v4.w;
            }
        } else {
#pragma unroll
            for (int u = 0; u < KPT; ++u) x[u] = (j0 + u < n) ? key[j0 + u] : 0u;
        }
        uint32_t ntake = 0;
#pragma unroll
        for (int u = 0; u < KPT; ++u) ntake += (j0 + u < n && x[u] >= tau) ? 1u : 0u;
        uint32_t tot;
        uint32_t pos = cnt + block_excl_sum(ntake, sm.warp_tot, tot);
        if (ntake) {
#pragma unroll
            for (int u = 0; u < KPT; ++u) {
                if (j0 + u < n && x[u] >= tau) {
                    if (pos < (uint32_t)TK_CAP) {
                        lk[pos] = x[u];
                        lj[pos] = (uint32_t)(j0 + u);
                    }
                    ++pos;
                }
            }
        }
        cnt += tot;
        __syncthreads();  // warp_tot is reused by the next step
    }
    if (cnt < (uint32_t)p.topk || cnt > (uint32_t)TK_CAP) {
        topk_exact_global(key, n, p.topk, orow, sm, srow);
        return;
    }

    // exact top K among the survivors, then an ordered keep (they are in j order)
    if (srow) {  // chunk mode also records the kept keys' scores
        uint32_t kth, need_eq;
        block_kth_shared(lk, (int)cnt, (uint32_t)p.topk, sm, kth, need_eq);
        __syncthreads();
        uint32_t eq_seen = 0, written = 0;
        for (int base = 0; base < (int)cnt; base += 4 * TK_THREADS) {
            const int e0 = base + 4 * tid;
            uint32_t x[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) x[u] = (e0 + u < (int)cnt) ? lk[e0 + u] : 0u;
            uint32_t neq = 0;
#pragma unroll
            for (int u = 0; u < 4; ++u) neq += (e0 + u < (int)cnt && x[u] == kth) ? 1u : 0u;
            uint32_t eq_tot;
            uint32_t eq_rank = eq_seen + block_excl_sum(neq, sm.warp_tot, eq_tot);
            bool take[4];
            uint32_t ntake = 0;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const bool valid = e0 + u < (int)cnt;
                const bool eq = valid && x[u] == kth;
                take[u] = (valid && x[u] > kth) || (eq && eq_rank < need_eq);
                eq_rank += eq ? 1u : 0u;
                ntake += take[u] ? 1u : 0u;
            }
            __syncthreads();
            uint32_t take_tot;
            uint32_t pos = written + block_excl_sum(ntake, sm.warp_tot2, take_tot);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (take[u]) {
                    srow[pos] = __uint_as_float(x[u]);
                    orow[pos++] = (int32_t)lj[e0 + u];
                }
            eq_seen += eq_tot;
            written += take_tot;
            __syncthreads();
        }
        return;
    }
    block_topk_ordered(lk, lj, (int)cnt, p.topk, orow, sm);
}

// The merge of a chunked row: one CTA per (sequence, group) row stages the
// chunks' lists (each ascending, chunks in order, so the whole is ascending in
// j) in shared memory as (score bits, j) and takes their exact top K, ties to
// the lower j.  The row's top K lies in the union of the chunks' top Ks.
__global__ void __launch_bounds__(TK_THREADS) k2_chunk_merge_kernel(Problem p, int n_chunks, int64_t chunk_len,
                                                                    const int32_t* __restrict__ cidx,
                                                                    const float* __restrict__ cscore,
                                                                    int32_t* __restrict__ idx) {
    __shared__ TopkSmem sm;
    __shared__ uint32_t chunk_cnt[32];
    extern __shared__ __align__(16) uint32_t mg_dyn[];
    const int K = p.topk;
    uint32_t* lk = mg_dyn;                      // [n_chunks * K] score bits
    uint32_t* lj = mg_dyn + n_chunks * K;       // [n_chunks * K] rows
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t row = blockIdx.x;             // b * H_kv + g
    int32_t* orow = idx + row * p.nq * K;       // one query per sequence
    // valid entries of each chunk (a prefix: -1 after)
    if (warp < n_chunks) {
        const int32_t* ir = cidx + (row * n_chunks + warp) * K;
        int c = 0;
        for (int u = lane; u < K; u += 32) c += ir[u] >= 0;
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (lane == 0) chunk_cnt[warp] = c;
    }
    __syncthreads();
    int total = 0;
    for (int c = 0; c < n_chunks; ++c) total += chunk_cnt[c];
    // stage the chunks' entries contiguously, in chunk order
    int base = 0;
    for (int c = 0; c < n_chunks; ++c) {
        const int cc = chunk_cnt[c];
        const int32_t* ir = cidx + (row * n_chunks + c) * K;
        const float* sr = cscore + (row * n_chunks + c) * K;
        for (int u = tid; u < cc; u += TK_THREADS) {
            lk[base + u] = __float_as_uint(sr[u]);
            lj[base + u] = (uint32_t)(ir[u] + c * chunk_len);
        }
        base += cc;
    }
    __syncthreads();
    if (total <= K) {
        for (int u = tid; u < K; u += TK_THREADS) orow[u] = u < total ? (int32_t)lj[u] : -1;
        return;
    }
    block_topk_ordered(lk, lj, total, K, orow, sm);
}

template <int D, int G>
cudaError_t launch_score_dg(const Problem& p, const void* q, const void* k, const float* lse, float* scores,
                            int i_begin, int i_count, int64_t sstride, cudaStream_t st) {
    constexpr int QPC = SC_WARPS * 2 * (8 / G);
    constexpr int SMEM = 2 * SC_BN * D * 2;
    auto kern = k2_score_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    // split the key range so that every (query block, group, sequence) gets
    // enough CTAs to fill the machine even for one query (decode)
    const int qblocks = (i_count + QPC - 1) / QPC;
    const int64_t t_hi = p.seq_len ? p.kv_len - 1 : p.q_pos0 + i_begin + i_count - 1;
    const int64_t cand = t_hi - p.window + 1;
    if (cand <= 0) return cudaSuccess;
    const int64_t work_ctas = (int64_t)qblocks * p.hkv * p.B;
    int64_t splits = (4 * 148 + work_ctas - 1) / work_ctas;
    const int64_t max_splits = (cand + 4 * SC_BN - 1) / (4 * SC_BN);
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    if (splits > 65535 / p.B) splits = 65535 / p.B;
    int64_t kps = (cand + splits - 1) / splits;
    kps = (kps + SC_BN - 1) / SC_BN * SC_BN;
    dim3 grid(qblocks, p.hkv, (unsigned)(p.B * splits));
    prof_begin(KID_SCORE, st);
    kern<<<grid, SC_WARPS * 32, SMEM, st>>>(p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, lse, scores,
                                            i_begin, i_count, sstride, kps, (int)splits);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_score_d(const Problem& p, const void* q, const void* k, const float* lse, float* scores,
                           int i_begin, int i_count, int64_t sstride, cudaStream_t st) {
    switch (p.hq / p.hkv) {
        case 1: return launch_score_dg<D, 1>(p, q, k, lse, scores, i_begin, i_count, sstride, st);
        case 2: return launch_score_dg<D, 2>(p, q, k, lse, scores, i_begin, i_count, sstride, st);
        case 4: return launch_score_dg<D, 4>(p, q, k, lse, scores, i_begin, i_count, sstride, st);
        default: return launch_score_dg<D, 8>(p, q, k, lse, scores, i_begin, i_count, sstride, st);
    }
}

}  // namespace

cudaError_t launch_score(const Problem& p, const void* q, const void* k, const float* lse, float* scores,
                         int i_begin, int i_count, int64_t sstride, cudaStream_t st) {
    if (p.D == 64) return launch_score_d<64>(p, q, k, lse, scores, i_begin, i_count, sstride, st);
    return launch_score_d<128>(p, q, k, lse, scores, i_begin, i_count, sstride, st);
}

cudaError_t launch_topk(const Problem& p, const float* scores, int64_t sstride, int32_t* idx, int i_begin,
                        int i_count, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(k2_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TK_DYN_SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(i_count, p.hkv, p.B);
    prof_begin(KID_TOPK, st);
    k2_topk_kernel<<<grid, TK_THREADS, TK_DYN_SMEM, st>>>(p, scores, sstride, idx, i_begin, i_count, 0, nullptr,
                                                          nullptr);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

// Decode rows (one query per sequence) that are too few to fill the SMs: each row
// is cut into key chunks (about two CTAs per SM in all), then merged per row.
void topk_chunk_geometry(const Problem& p, int64_t n_cand_max, int64_t& chunk_len, int& n_chunks) {
    const int64_t rows = (int64_t)p.B * p.hkv;
    chunk_len = 0;
    n_chunks = 1;
    if (p.nq != 1 || rows > 74 || n_cand_max < 4 * TK_CAP) return;
    int want = (int)(2 * 148 / rows);
    if (want > 16) want = 16;
    if (want < 2) return;
    int64_t len = (n_cand_max + want - 1) / want;
    if (len < TK_CAP) len = TK_CAP;
    len = (len + 3) / 4 * 4;  // chunks start on 16-byte boundaries of the score rows
    const int nc = (int)((n_cand_max + len - 1) / len);
    if (nc < 2) return;
    chunk_len = len;
    n_chunks = nc;
}

size_t topk_chunk_bytes(const Problem& p, int64_t n_cand_max) {
    int64_t len;
    int nc;
    topk_chunk_geometry(p, n_cand_max, len, nc);
    if (nc < 2) return 0;
    return (size_t)nc * p.B * p.hkv * p.topk * 8 + 256;
}

cudaError_t launch_topk_decode(const Problem& p, const float* scores, int64_t sstride, int64_t n_cand_max,
                               int32_t* idx, void* chunk_scratch, cudaStream_t st) {
    int64_t len;
    int nc;
    topk_chunk_geometry(p, n_cand_max, len, nc);
    if (nc < 2 || chunk_scratch == nullptr) return launch_topk(p, scores, sstride, idx, 0, 1, st);
    cudaError_t e = cudaFuncSetAttribute(k2_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TK_DYN_SMEM);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)p.B * p.hkv;
    int32_t* cidx = reinterpret_cast<int32_t*>(chunk_scratch);
    float* cscore = reinterpret_cast<float*>(cidx + (size_t)nc * rows * p.topk);
    prof_begin(KID_TOPK, st);
    k2_topk_kernel<<<dim3(nc, p.hkv, p.B), TK_THREADS, TK_DYN_SMEM, st>>>(p, scores, sstride, idx, 0, 1, len, cidx,
                                                                         cscore);
    prof_end(st);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int smem = nc * p.topk * 8;  // at most 16 x 2048 x 8 = 256 KB: nc * topk <= 16384 is required
    if (smem > 200 * 1024) return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(k2_chunk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
        return e;
    prof_begin(KID_TOPK, st);
    k2_chunk_merge_kernel<<<(unsigned)rows, TK_THREADS, smem, st>>>(p, nc, len, cidx, cscore, idx);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

}  // namespace hs2
