// k2_select_tc.cu -- K2 on the tensor cores: HySparse2's token-level
// selection (xiawanshe.com report, section "Token级选择": per token, the 1024
// best older tokens beside the forced 128-token window; davidyin.dev notes,
// section "HySparse2 的解法": no separate indexer, so the score comes from the
// full-attention layer's own probabilities).
//
//   score_{g,j}(t) = sum_{h in g} 2^(s2_{h,j} - lse2_h),  s2 = scale*log2(e)*<q_h, k_j>
//
// One CTA = one KV group x QT consecutive queries (N = QT*G columns ordered
// (query, head)); it sweeps the candidate keys in 128-key tiles:
//   S^T (TMEM, 128 keys x N, double buffered) = K_tile Q^T    tcgen05.mma
// and the epilogue thread that owns TMEM lane r (= key j) forms the group sum
// for each of its queries inside one thread.  Three passes keep the work on
// chip and exact:
//   SAMPLE  1024 keys at a fixed stride S = kv_len / 1024 over the whole cache
//           (a strided tensor-map view, 8 tiles of 128): sample scores spread
//           over every segment of the context, not a few contiguous runs
//   (k2_thresh_kernel) per row, a bound tau that at least K candidates
//           exceed with high probability: the r-th largest sample, r = L +
//           4.5 sqrt(L) + 2, where L = K s/n is the expected number of samples
//           above the K-th best candidate
//   FILTER  every tile; candidates at or above the row's bound are appended
//           to the row's survivor list in this SM's slot of the workspace
//           (L2-resident).  A list about to overflow is compacted in place to
//           its exact top K and the bound is raised to its K-th entry.  At the
//           end each row's exact top-min(K, n) is taken from the list (radix
//           select on the fp32 bits, ties to the lower j, output ascending) --
//           or, if fewer than min(K, n) candidates passed (tau overestimated),
//           the row is marked,
//   RETRY   re-runs only the tiles with a marked row, with bound 0.
// Ties: every exact select keeps, among the entries equal to the K-th score,
// those with the lowest j (a second radix pass on j when the tie straddles
// the cut).  The exact select can also write each selected key's score (used
// to merge the selections of several slices of one context).
//
// Two layouts of the epilogue share everything else (the MMA, TMA, score
// math and exact selects):
//   ORDERED  32 queries per CTA on 4 warpgroups of 8 queries.  Each tile, the
//            four warps of a warpgroup exchange their per-row counts, so the
//            survivors are appended in ascending j and the final select
//            writes them out in list order.
//   COUNTER  28 queries per CTA on 7 warpgroups of 4 queries.  A survivor
//            takes its position from the row's shared counter (one shared
//            atomic per key that passes): a tile's entries land in any order,
//            tiles stay in order, and the final select ranks each kept entry
//            inside its tile's run.
// ORDERED serves short candidate ranges, whose rows keep many survivors
// (about 12% of the candidates at a 32K context); COUNTER serves long ones
// (under 1% at 1M), where its 28 warps hide more latency and 28-query CTAs
// fill the last wave of a 4096-query chunk (588 CTAs = 3.97 waves of 148 SMs
// against 512 = 3.46).
//
// The same sweep in MODE_BLOCK serves block-level selection (the design
// token-level selection replaces, same report and section): the epilogue sums
// each warp's 32 keys per query and writes one float per 32 candidate keys,
// and k2_block_topk_kernel ranks whole blocks from those sums.  It takes the
// token sweep's geometry for the same candidate count (ORDERED or COUNTER).
//
// The buffer may hold one slice of a longer context (context parallelism):
// positions are then shifted by the slice's first key, and every candidate
// range is cut at the slice's last key (last_cand).
#include <cudaTypedefs.h>

#include "hs2_kernels.h"
#include "tc05.cuh"

namespace hs2 {

bool make_map(CUtensorMap* m, const void* base, uint64_t x, uint64_t y, uint64_t z, uint32_t box_rows);  // k1_full_tc.cu
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();                                      // k1_full_tc.cu

namespace {

constexpr int SL_BN = 128;         // keys per tile (MMA M)
constexpr int SL_NS = 3;           // K pipeline stages
constexpr int SL_SAMPLE_TILES = 8; // sample tiles per CTA
constexpr int SL_SPR = SL_SAMPLE_TILES * SL_BN;  // sample slots per row
constexpr int SL_CMAX = 4096;      // survivor list capacity per row
constexpr int SL_SLOTS = 256;      // per-SM survivor slots (indexed by %smid)
constexpr int SL_MIN_SMEM = 120 * 1024;  // keeps one CTA per SM (slots are per SM)
constexpr int SL_STAGE = 1024;     // COUNTER final select: one row's kept keys per warp in shared memory
constexpr int64_t SL_COUNTER_MIN_CAND = int64_t(1) << 18;  // calls whose longest row has this many
                                                           // candidates use the COUNTER layout

enum { MODE_SAMPLE = 0, MODE_FILTER = 1, MODE_RETRY = 2, MODE_BLOCK = 3 };
enum { ORDERED = 0, COUNTER = 1 };

template <int L>
struct Lay;
template <>
struct Lay<ORDERED> {
    static constexpr int QT = 32, EPI_WARPS = 16;
};
template <>
struct Lay<COUNTER> {
    static constexpr int QT = 28, EPI_WARPS = 28;
};

// COUNTER's MMA has N = 28 G columns: a valid M = 128 shape (a multiple of 16)
// only for G of 4 and 8.  Calls with G of 1 or 2 keep ORDERED (N = 32 G) at
// every length.
template <int G>
constexpr bool kCounterFits = (Lay<COUNTER>::QT * G) % 16 == 0;

template <int D, int G, int L>
struct SlCfg {
    static constexpr int QT = Lay<L>::QT;               // queries per CTA
    static constexpr int EPI_WARPS = Lay<L>::EPI_WARPS;  // epilogue warps
    static constexpr int NWG = EPI_WARPS / 4;           // warpgroups, each 1/NWG of the query columns
    static constexpr int QH = QT / NWG;                 // queries of one warpgroup
    static constexpr int TMA_WARP = EPI_WARPS, MMA_WARP = EPI_WARPS + 1;
    static constexpr int THREADS = 32 * (EPI_WARPS + 2);
    static constexpr int N = QT * G;               // MMA N: (query, head) columns
    static constexpr int KB = D / 64;
    static constexpr int QBLK = N * 128;           // one 64-wide column block of Q (N rows x 128 B)
    static constexpr int KBLK = SL_BN * 128;       // one 64-wide column block of a K tile
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + KB * QBLK;
    static constexpr int K_END = K_OFF + SL_NS * KB * KBLK;
    // COUNTER: after the sweep, the final select stages each row's kept keys over
    // the dead Q tile and K ring, SL_STAGE int32 per epilogue warp
    static constexpr int STAGE_BYTES = L == COUNTER ? EPI_WARPS * SL_STAGE * 4 : 0;
    static constexpr int MISC_OFF = K_END > STAGE_BYTES ? K_END : STAGE_BYTES;
    // misc: barriers, l2[N], row state, per-warp histograms and counts
    static constexpr int BAR_BYTES = 256;
    static constexpr int L2_OFF = MISC_OFF + BAR_BYTES;
    static constexpr int ROW_OFF = L2_OFF + N * 4;
    static constexpr int ROW_BYTES = QT * 5 * 4 + 32;    // cnt[2], lo, tlim, act; per-warpgroup ovf
    static constexpr int WCNT_OFF = ROW_OFF + ROW_BYTES;  // ORDERED: [4 warps][QT rows]
    static constexpr int HIST_OFF = WCNT_OFF + 4 * QT * 4;
    static constexpr int END = HIST_OFF + EPI_WARPS * 256 * 4;
    static constexpr int SMEM_NEED = END + 1024;
    static constexpr int SMEM = SMEM_NEED > SL_MIN_SMEM ? SMEM_NEED : SL_MIN_SMEM;
    static constexpr uint32_t TMEM_COLS = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128 : (2 * N <= 256) ? 256 : 512;
    static_assert(NWG <= 8, "named barriers 1..NWG");
    static_assert(QT % NWG == 0, "whole queries per warpgroup");
    static_assert(N % 16 == 0 && N <= 256, "MMA N of an M = 128 tcgen05.mma: a multiple of 16, at most 256");
    static_assert(N / NWG >= 8, "a warpgroup's columns fill one tensor-memory load of at least 8 columns");
};

enum : int { SB_Q = 0, SB_KFULL = 1, SB_KEMPTY = SB_KFULL + SL_NS, SB_SFULL = SB_KEMPTY + SL_NS,
             SB_SEMPTY = SB_SFULL + 2, SB_DRAIN = SB_SEMPTY + 2, SB_COUNT = SB_DRAIN + 1 };

struct SelArgs {
    const float* lse;       // [B, H_q, n_q]
    int32_t* idx;           // [B, H_kv, n_q, K]
    float* samples;         // [rows][SL_SPR]
    int32_t* s_valid;       // [rows] valid samples per row
    float* tau;             // [rows] threshold estimate
    int32_t* status;        // [rows] 1 = needs the retry pass, 2 = selected by it
    uint2* slots;           // [n_slots][QT][cmax] (score bits, j)
    int i_begin, i_count;   // query chunk of this call
    int cmax;               // survivor list capacity per row
    int slot_by_block;      // 1: slot = block id (small grids); 0: slot = %smid (one CTA per SM)
    int64_t sample_stride;  // S: the sampling pass reads keys 0, S, 2S, ...
    float* csum;            // block mode: [rows][cstride] sums of 32 consecutive candidate scores
    int64_t cstride;
    float* sel_score;       // optional [B, H_kv, n_q, K]: the score of every selected key (-1 padding)
};

// Last candidate key of the query at t: t - window, and not past the buffer's
// last key (when the buffer holds one slice of a longer context, a query may
// sit past its end, or before its start: then it has no candidate here).
__device__ __forceinline__ int64_t last_cand(const Problem& p, int64_t t) {
    return min(t - p.window, p.kv_len - 1);
}

__device__ __forceinline__ uint32_t smid() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%smid;\n" : "=r"(r));
    return r;
}

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n)); }

// ---------------------------------------------------------------------------
// warp-level exact selection on (score bits, j) lists

// The K-th largest key among the keys key(i) of the entries i < n that key()
// accepts (8-bit radix, four passes, one warp): kth, how many entries equal to
// kth belong to the top K (need_eq), and how many equal kth in all (eq_total).
// K must not exceed the number of accepted entries.
template <class KeyFn>
__device__ void warp_radix_kth(int n, uint32_t K, uint32_t* hist, KeyFn key, uint32_t& kth, uint32_t& need_eq,
                               uint32_t& eq_total) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, pmask = 0, k_rem = K, in_bin = 0;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int u = lane; u < 256; u += 32) hist[u] = 0;
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
            uint32_t x;
            if (key(i, x) && (x & pmask) == prefix) atomicAdd(&hist[(x >> shift) & 255u], 1u);
        }
        __syncwarp();
        uint32_t bins[8], s = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            bins[u] = hist[8 * (31 - lane) + u];
            s += bins[u];
        }
        uint32_t incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - s;
        uint32_t digit = 0, krem_new = 0, cnt = 0;
        const bool mine = excl < k_rem && k_rem <= incl;
        if (mine) {
            uint32_t above = excl;
#pragma unroll
            for (int u = 7; u >= 0; --u) {
                if (above + bins[u] >= k_rem) {
                    digit = 8 * (31 - lane) + u;
                    krem_new = k_rem - above;
                    cnt = bins[u];
                    break;
                }
                above += bins[u];
            }
        }
        const uint32_t who = __ballot_sync(0xffffffffu, mine);
        const int src = who ? __ffs(who) - 1 : 0;
        digit = __shfl_sync(0xffffffffu, digit, src);
        krem_new = __shfl_sync(0xffffffffu, krem_new, src);
        in_bin = __shfl_sync(0xffffffffu, cnt, src);
        prefix |= digit << shift;
        pmask |= 255u << shift;
        k_rem = krem_new;
        __syncwarp();
    }
    kth = prefix;
    need_eq = k_rem;
    eq_total = in_bin;
}

// The K-th largest of the first n keys of `key` (element stride `stride`).
__device__ void warp_kth(const uint32_t* key, int stride, int n, uint32_t K, uint32_t* hist, uint32_t& kth,
                         uint32_t& need_eq) {
    uint32_t eq_total;
    warp_radix_kth(
        n, K, hist,
        [&](int i, uint32_t& x) {
            x = key[(int64_t)i * stride];
            return true;
        },
        kth, need_eq, eq_total);
}

// The exact top K of a survivor list under the order (score desc, j asc): the
// K-th score kth, and jth, the largest j kept among the entries whose score
// equals kth (the need_eq smallest such j; all of them when none is left out).
// The list's j are distinct.  Keeping the entries with score > kth, or score
// == kth and j <= jth, keeps exactly K.
__device__ void list_topk_bound(const uint2* list, int n, uint32_t K, uint32_t* hist, uint32_t& kth, uint32_t& jth) {
    uint32_t need_eq, eq_total;
    warp_radix_kth(
        n, K, hist,
        [&](int i, uint32_t& x) {
            x = list[i].x;
            return true;
        },
        kth, need_eq, eq_total);
    jth = 0xffffffffu;
    if (eq_total > need_eq) {  // ties at the K-th score straddle the cut: keep the lowest j
        const uint32_t k_ = kth;
        uint32_t njth, ne2, eq2;
        warp_radix_kth(
            n, need_eq, hist,
            [&](int i, uint32_t& x) {
                const uint2 e = list[i];
                x = ~e.y;
                return e.x == k_;
            },
            njth, ne2, eq2);
        jth = ~njth;
    }
}

__device__ __forceinline__ bool kept(uint2 e, uint32_t kth, uint32_t jth) {
    return e.x > kth || (e.x == kth && e.y <= jth);
}

// Keep, in list order, the entries that list_topk_bound's (kth, jth) keeps,
// compacted in place to the front of `list`; with `stage`, their j are also
// written to stage[0..kept).  Returns the number kept.
__device__ int warp_compact(uint2* list, int n, uint32_t kth, uint32_t jth, int32_t* stage = nullptr) {
    const int lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t written = 0;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        uint2 e = make_uint2(0u, 0u);
        if (i < n) e = list[i];
        const bool take = i < n && kept(e, kth, jth);
        const uint32_t tb = __ballot_sync(0xffffffffu, take);
        const uint32_t pos = written + __popc(tb & lt);
        __syncwarp();
        if (take) {
            list[pos] = e;
            if (stage) stage[pos] = (int32_t)e.y;
        }
        written += __popc(tb);
    }
    __syncwarp();
    return (int)written;
}

// The kept entries' j (and, if sout is not null, their scores) written to out
// in list order.  Returns the number written.
__device__ int warp_take(const uint2* list, int n, uint32_t kth, uint32_t jth, int32_t* out, float* sout) {
    const int lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t written = 0;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        uint2 e = make_uint2(0u, 0u);
        if (i < n) e = list[i];
        const bool take = i < n && kept(e, kth, jth);
        const uint32_t tb = __ballot_sync(0xffffffffu, take);
        if (take) {
            const uint32_t pos = written + __popc(tb & lt);
            out[pos] = (int32_t)e.y;
            if (sout) sout[pos] = __uint_as_float(e.x);
        }
        written += __popc(tb);
    }
    __syncwarp();
    return (int)written;
}

// The selection of one row, ascending by j, from its kept entries list[0..n),
// ordered by key tile (j / SL_BN) but in any order inside a tile; their j are
// read through jat(i) (a staged copy in shared memory, or the list itself).
// An entry's output position is the number of kept entries in earlier tiles
// -- the start of its tile's run -- plus its rank by j inside the run.
// Writes out[0..n) and, if sout is not null, the scores beside them.
template <class JFn>
__device__ void warp_emit_sorted(const uint2* list, int n, JFn jat, int32_t* out, float* sout) {
    const int lane = threadIdx.x & 31;
    for (int i = lane; i < n; i += 32) {
        const int32_t j = jat(i);
        const int32_t tile = j / SL_BN;
        int lo = i, hi = i + 1;
        while (lo > 0 && jat(lo - 1) / SL_BN == tile) --lo;
        while (hi < n && jat(hi) / SL_BN == tile) ++hi;
        int rank = 0;
        for (int u = lo; u < hi; ++u) rank += jat(u) < j;
        out[lo + rank] = j;
        if (sout) sout[lo + rank] = __uint_as_float(list[i].x);
    }
}

// ---------------------------------------------------------------------------

template <int D, int G, int MODE, int L>
__global__ void __launch_bounds__(SlCfg<D, G, L>::THREADS, 1)
    k2_select_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, Problem p,
                        SelArgs a) {
    using C = SlCfg<D, G, L>;
    constexpr int N = C::N;
    constexpr int QT = C::QT;
    constexpr int NH = N / C::NWG;           // columns of one epilogue warpgroup
    constexpr int CW = NH < 32 ? NH : 32;    // columns per TMEM load
    constexpr int QH = C::QH;                // queries of one epilogue warpgroup
    static_assert(NH % CW == 0 && CW % G == 0, "whole queries per TMEM load");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
    const uint32_t sQ = sbase + C::Q_OFF, sK = sbase + C::K_OFF;
    const uint32_t bars = sbase + C::MISC_OFF;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + C::MISC_OFF + 8 * SB_COUNT);
    tc::Abort* ab = reinterpret_cast<tc::Abort*>(sgen + C::MISC_OFF + 8 * SB_COUNT + 8);
    volatile int* okv = reinterpret_cast<volatile int*>(sgen + C::MISC_OFF + 8 * SB_COUNT + 16);  // [wg][2]
    float* l2s = reinterpret_cast<float*>(sgen + C::L2_OFF);
    // ORDERED: r_cnt[tile parity][QT] list lengths; COUNTER: r_cnt[QT], the rows' counters
    int32_t* r_cnt = reinterpret_cast<int32_t*>(sgen + C::ROW_OFF);
    float* r_lo = reinterpret_cast<float*>(r_cnt + 2 * QT);   // keep scores >= r_lo
    int32_t* r_tlim = reinterpret_cast<int32_t*>(r_lo + QT);  // last candidate key of the row
    int32_t* r_act = r_tlim + QT;                             // row takes part in this pass
    // COUNTER, per warpgroup: the last tile after which one of its rows passed the
    // compaction threshold (written by the appending lanes)
    volatile int32_t* r_ovf = r_act + QT;
    int32_t* wcnt = reinterpret_cast<int32_t*>(sgen + C::WCNT_OFF);    // ORDERED: [4 key quarters][QT rows]
    uint32_t* hist = reinterpret_cast<uint32_t*>(sgen + C::HIST_OFF);  // [epilogue warps][256]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * QT;  // first query of the CTA within the chunk
    const int nq_here = min(QT, a.i_count - q0);
    const int64_t pos0 = seq_pos0(p, b, KID_SCORE) + a.i_begin;
    const int64_t t_max = pos0 + q0 + nq_here - 1;
    const int64_t cand_end = last_cand(p, t_max) + 1;  // candidate keys are j < cand_end
    const int64_t row0 = (int64_t)(b * p.hkv + g) * a.i_count + q0;  // chunk row of query q0
    if (cand_end <= 0 && MODE != MODE_FILTER) return;
    const int n_ct = cand_end > 0 ? (int)((cand_end + SL_BN - 1) / SL_BN) : 0;

    if (MODE == MODE_RETRY) {
        // only tiles with a row marked by the filter pass run again
        int need = 0;
        for (int q = 0; q < nq_here; ++q) need |= a.status[row0 + q];
        if (!need) return;
    }
    const uint32_t slot = a.slot_by_block ? (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x : smid();
    if ((MODE == MODE_FILTER || MODE == MODE_RETRY) && slot >= SL_SLOTS) {
        if (tid == 0) report_error(p.err, HS2_ERR_DEVICE_CHECK, KID_SCORE, slot, 0);
        return;
    }
    const int cmax = a.cmax;
    // a row whose list grew past thr is compacted to its exact top K before the
    // next tile (which adds at most SL_BN entries); cmax >= topk + SL_BN unless
    // cmax holds every candidate of the call
    const int thr = max(cmax - SL_BN, p.topk);
    uint2* lists = a.slots + (int64_t)slot * QT * cmax;
    // sampling pass: tile it holds keys S (128 it + u), u < 128, of the strided view
    const int64_t S = a.sample_stride;
    const int64_t n_sb = cand_end > 0 ? (cand_end + S - 1) / S : 0;  // sampled keys below the candidate limit
    const int n_tiles = MODE == MODE_SAMPLE ? (int)min((int64_t)SL_SAMPLE_TILES, (n_sb + SL_BN - 1) / SL_BN) : n_ct;

    // row state
    if (tid < QT) {
        const int q = tid;
        const bool live = q < nq_here;
        const int64_t t = pos0 + q0 + q;
        const int64_t n = last_cand(p, t) + 1;
        float bs = 0.f;
        int32_t act = live && n > 0;
        if (MODE == MODE_FILTER && act) bs = a.tau[row0 + q];
        if (MODE == MODE_RETRY) act = live && a.status[row0 + q] != 0;
        r_cnt[q] = 0;
        r_cnt[QT + q] = 0;
        if (q < C::NWG) r_ovf[q] = -1;
        r_lo[q] = act ? bs : INFINITY;
        r_tlim[q] = (int32_t)max(last_cand(p, t), (int64_t)-1);
        r_act[q] = act;
    }
    for (int c = tid; c < N; c += C::THREADS) {
        const int q = c / G, hh = c % G;
        const int i = a.i_begin + q0 + q;
        l2s[c] = (q < nq_here) ? a.lse[(int64_t)(b * p.hq + g * G + hh) * p.nq + i] * kLog2e : INFINITY;
    }
    if (tid == 0) {
        for (int i = 0; i < SB_COUNT; ++i)
            tc::mbar_init(bar(i), (i >= SB_SEMPTY && i < SB_SEMPTY + 2) ? 32 * C::EPI_WARPS : 1);
        ab->flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == C::MMA_WARP) tc::tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == C::TMA_WARP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n_tiles > 0) {
            tc::mbar_expect_tx(bar(SB_Q), C::KB * C::QBLK);
            for (int kb = 0; kb < C::KB; ++kb)
                tc::tma_load_4d(sQ + kb * C::QBLK, &tm_q, bar(SB_Q), kb * 64, g * G, a.i_begin + q0, b);
            int issued = 0;
            for (int it = 0; it < n_tiles; ++it) {
                const int s = it % SL_NS;
                if (it >= SL_NS && !tc::mbar_wait(bar(SB_KEMPTY + s), ((it - SL_NS) / SL_NS) & 1, ab, p.err, KID_SCORE, 1))
                    break;
                tc::mbar_expect_tx(bar(SB_KFULL + s), C::KB * C::KBLK);
                const int kt = it;
                for (int kb = 0; kb < C::KB; ++kb)
                    tc::tma_load_3d(sK + (s * C::KB + kb) * C::KBLK, &tm_k, bar(SB_KFULL + s), kb * 64, kt * SL_BN,
                                    b * p.hkv + g);
                issued = it + 1;
            }
            if (ab->flag) {
                tc::Abort none{0};
                tc::mbar_wait(bar(SB_Q), 0, &none, nullptr, 0, 0);
                for (int it = (issued > SL_NS ? issued - SL_NS : 0); it < issued; ++it)
                    tc::mbar_wait(bar(SB_KFULL + it % SL_NS), (it / SL_NS) & 1, &none, nullptr, 0, 0);
            }
        }
    } else if (warp == C::MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t ID = tc::idesc_bf16(SL_BN, N, 0, 0);
            bool ok = tc::mbar_wait(bar(SB_Q), 0, ab, p.err, KID_SCORE, 2);
            for (int it = 0; ok && it < n_tiles; ++it) {
                const int s = it % SL_NS, sb = it & 1;
                ok = tc::mbar_wait(bar(SB_KFULL + s), (it / SL_NS) & 1, ab, p.err, KID_SCORE, 3);
                if (ok && it >= 2) ok = tc::mbar_wait(bar(SB_SEMPTY + sb), ((it - 2) >> 1) & 1, ab, p.err, KID_SCORE, 4);
                if (!ok) break;
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t da = tc::sdesc_sw128(sK + (s * C::KB + (kk >> 2)) * C::KBLK + (kk & 3) * 32, 16, 1024);
                    const uint64_t db = tc::sdesc_sw128(sQ + (kk >> 2) * C::QBLK + (kk & 3) * 32, 16, 1024);
                    tc::mma_ss(tmem + sb * N, da, db, ID, kk > 0);
                }
                tc::mma_commit(bar(SB_SFULL + sb));
                tc::mma_commit(bar(SB_KEMPTY + s));
            }
            tc::mma_commit(bar(SB_DRAIN));
            tc::Abort none{0};
            tc::mbar_wait(bar(SB_DRAIN), 0, &none, nullptr, 0, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue warps
        // warp w reads TMEM lanes 32*(w%4).. (keys of quarter kq) and the columns of
        // warpgroup wg = w/4 (queries QH*wg .. QH*wg+QH-1)
        const int wg = warp >> 2, kq = warp & 3;
        const int et = tid & 127;  // key lane within the tile
        const uint32_t lane_off = (uint32_t)(kq * 32) << 16;
        const int barid = 1 + wg;
        bool ok = true;
        float lo[QH];
        int32_t tlim[QH];
#pragma unroll
        for (int qq = 0; qq < QH; ++qq) {
            lo[qq] = r_lo[wg * QH + qq];
            tlim[qq] = r_tlim[wg * QH + qq];
        }
        for (int it = 0; it < n_tiles; ++it) {
            const int sb = it & 1;
            const int64_t jb = (int64_t)it * SL_BN;
            const int64_t j = MODE == MODE_SAMPLE ? S * (jb + et) : jb + et;
            // one thread per warpgroup waits (bounded) and the named barrier hands
            // the result to its four warps, so they leave the loop together
            if (et == 0) okv[wg * 2 + (it & 1)] = tc::mbar_wait(bar(SB_SFULL + sb), (it >> 1) & 1, ab, p.err, KID_SCORE, 5);
            named_sync(barid, 128);
            if (!okv[wg * 2 + (it & 1)]) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            if constexpr (MODE == MODE_FILTER || MODE == MODE_RETRY) {
                // rare: a row whose list could overflow on this tile is first cut to its
                // exact top K; later keys (larger j) then need a score strictly above its
                // K-th entry.  The four warps of a warpgroup take the same decision:
                //   ORDERED  from this tile's counts, which no warp changes before the
                //            warpgroup's next barrier (the next tile's go to the other slot);
                //   COUNTER  from the warpgroup's mark, written before this tile's barrier
                //            and changed by no warp of the warpgroup before it decides.
                int32_t* cnt_now = r_cnt + (L == ORDERED ? (it & 1) * QT : 0);
                bool need = false;
                if constexpr (L == ORDERED) {
#pragma unroll
                    for (int qq = 0; qq < QH; ++qq) need |= cnt_now[wg * QH + qq] > thr;
                } else {
                    need = r_ovf[wg] == it - 1;
                }
                if (need) {
                    named_sync(barid, 128);
#pragma unroll 1
                    for (int qq = kq; qq < QH; qq += 4) {
                        const int q = wg * QH + qq;
                        const int cnt = min(cnt_now[q], cmax);  // only this warp changes it now
                        if (cnt <= thr) continue;
                        uint2* lst = lists + (int64_t)q * cmax;
                        uint32_t kth, jth;
                        list_topk_bound(lst, cnt, (uint32_t)p.topk, hist + warp * 256, kth, jth);
                        const int kept = warp_compact(lst, cnt, kth, jth);
                        if (lane == 0) {
                            cnt_now[q] = kept;
                            r_lo[q] = nextafterf(__uint_as_float(kth), INFINITY);
                        }
                    }
                    named_sync(barid, 128);
#pragma unroll
                    for (int qq = 0; qq < QH; ++qq) lo[qq] = r_lo[wg * QH + qq];
                }
            }
            float sc[QH];
#pragma unroll
            for (int c = 0; c < NH / CW; ++c) {
                float v[CW];
                const uint32_t col = sb * N + wg * NH + c * CW;
                if constexpr (CW == 32) tc::tmem_ld32(tmem + lane_off + col, v);
                else if constexpr (CW == 16) tc::tmem_ld16(tmem + lane_off + col, v);
                else tc::tmem_ld8(tmem + lane_off + col, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int qq = 0; qq < CW / G; ++qq) {
                    // p_h = 2^(s2 - lse2) for the G heads, summed as a tree
                    float e[G], lv[G];
                    const float* lrow = l2s + wg * NH + c * CW + qq * G;
                    if constexpr (G % 4 == 0) {
#pragma unroll
                        for (int h4 = 0; h4 < G / 4; ++h4) {
                            const float4 x = reinterpret_cast<const float4*>(lrow)[h4];
                            lv[4 * h4] = x.x; lv[4 * h4 + 1] = x.y; lv[4 * h4 + 2] = x.z; lv[4 * h4 + 3] = x.w;
                        }
                    } else {
#pragma unroll
                        for (int hh = 0; hh < G; ++hh) lv[hh] = lrow[hh];
                    }
#pragma unroll
                    for (int hh = 0; hh < G; ++hh) e[hh] = ex2(fmaf(v[qq * G + hh], p.scale_log2, -lv[hh]));
#pragma unroll
                    for (int w2 = 1; w2 < G; w2 *= 2)
#pragma unroll
                        for (int hh = 0; hh + w2 < G; hh += 2 * w2) e[hh] += e[hh + w2];
                    sc[c * (CW / G) + qq] = e[0];
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(bar(SB_SEMPTY + sb));

            if constexpr (MODE == MODE_BLOCK) {
                // sum of the warp's 32 keys for each of its QH queries, as a transposing
                // butterfly: every exchange halves the values a lane holds, so lane l ends
                // with query l / (32 / QH) summed over all 32 lanes.  Both layouts add the
                // lanes in the same tree (xor 16, 8, 4, 2, 1), so their sums agree bit for bit.
                static_assert(QH == 8 || QH == 4, "the butterflies below reduce 8 or 4 query columns");
                float h1;
                const bool b4 = lane & 16, b3 = lane & 8;
                if constexpr (QH == 8) {
                    float h4[4], h2[2];
                    const bool b2 = lane & 4;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        h4[u] = (b4 ? sc[4 + u] : sc[u]) + __shfl_xor_sync(0xffffffffu, b4 ? sc[u] : sc[4 + u], 16);
#pragma unroll
                    for (int u = 0; u < 2; ++u)
                        h2[u] = (b3 ? h4[2 + u] : h4[u]) + __shfl_xor_sync(0xffffffffu, b3 ? h4[u] : h4[2 + u], 8);
                    h1 = (b2 ? h2[1] : h2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? h2[0] : h2[1], 4);
                } else {
                    float h2[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u)
                        h2[u] = (b4 ? sc[2 + u] : sc[u]) + __shfl_xor_sync(0xffffffffu, b4 ? sc[u] : sc[2 + u], 16);
                    h1 = (b3 ? h2[1] : h2[0]) + __shfl_xor_sync(0xffffffffu, b3 ? h2[0] : h2[1], 8);
                    h1 += __shfl_xor_sync(0xffffffffu, h1, 4);
                }
                h1 += __shfl_xor_sync(0xffffffffu, h1, 2);
                h1 += __shfl_xor_sync(0xffffffffu, h1, 1);
                constexpr int LPQ = 32 / QH;  // lanes per query after the exchanges
                const int q = wg * QH + lane / LPQ;
                if (lane % LPQ == 0 && q < nq_here)
                    a.csum[(row0 + q) * a.cstride + (jb >> 5) + kq] = h1;
            } else if constexpr (MODE == MODE_SAMPLE) {
#pragma unroll
                for (int qq = 0; qq < QH; ++qq) {
                    const int q = wg * QH + qq;
                    if (q < nq_here) {
                        const int64_t t = pos0 + q0 + q;
                        a.samples[(row0 + q) * SL_SPR + it * SL_BN + et] = (j <= last_cand(p, t)) ? sc[qq] : 0.f;
                    }
                }
            } else if constexpr (L == ORDERED) {
                // FILTER / RETRY, ORDERED: append in ascending j of the candidates at or
                // above each row's bound; key quarter kq's entries follow quarters < kq.
                // Tiles entirely below every row's candidate limit skip the per-row test.
                const bool all_valid = (int64_t)jb + SL_BN - 1 <= last_cand(p, pos0 + q0);
                const uint32_t lt = (1u << lane) - 1u;
                uint32_t bal[QH];
#pragma unroll
                for (int qq = 0; qq < QH; ++qq) {
                    bool keep = sc[qq] >= lo[qq];
                    if (!all_valid) keep = keep && (int32_t)j <= tlim[qq];
                    bal[qq] = __ballot_sync(0xffffffffu, keep);
                }
                if (lane < QH) {
                    uint32_t mine = 0;
#pragma unroll
                    for (int qq = 0; qq < QH; ++qq) mine = (lane == qq) ? bal[qq] : mine;
                    wcnt[kq * QT + wg * QH + lane] = __popc(mine);
                }
                named_sync(barid, 128);
                // lane qq: base position of row (wg, qq) for this warp's key quarter; the
                // last quarter's warp publishes the row's new count for the next tile
                int mybase = 0;
                if (lane < QH) {
                    const int q = wg * QH + lane;
                    mybase = r_cnt[(it & 1) * QT + q];
                    for (int w = 0; w < kq; ++w) mybase += wcnt[w * QT + q];
                    if (kq == 3) r_cnt[((it + 1) & 1) * QT + q] = mybase + wcnt[3 * QT + q];
                }
#pragma unroll
                for (int qq = 0; qq < QH; ++qq) {
                    const int pos = __shfl_sync(0xffffffffu, mybase, qq) + __popc(bal[qq] & lt);
                    if (((bal[qq] >> lane) & 1u) && pos < cmax)
                        lists[(wg * QH + qq) * cmax + pos] = make_uint2(__float_as_uint(sc[qq]), (uint32_t)j);
                }
            } else {
                // FILTER / RETRY, COUNTER: a candidate at or above its row's bound takes
                // the next position of the row's list from the row's shared counter (a
                // tile's entries in any order, tiles in ascending order); a row that passes
                // thr marks the warpgroup, and the next tile starts by compacting it.
                const bool all_valid = (int64_t)jb + SL_BN - 1 <= last_cand(p, pos0 + q0);
                bool keep[QH];
                int pos[QH];
#pragma unroll
                for (int qq = 0; qq < QH; ++qq) {
                    keep[qq] = sc[qq] >= lo[qq];
                    if (!all_valid) keep[qq] = keep[qq] && (int32_t)j <= tlim[qq];
                    pos[qq] = keep[qq] ? atomicAdd(&r_cnt[wg * QH + qq], 1) : cmax;
                }
#pragma unroll
                for (int qq = 0; qq < QH; ++qq) {
                    if (pos[qq] < cmax)
                        lists[(int64_t)(wg * QH + qq) * cmax + pos[qq]] =
                            make_uint2(__float_as_uint(sc[qq]), (uint32_t)j);
                    if (keep[qq] && pos[qq] >= thr) r_ovf[wg] = it;
                }
            }
        }
        if constexpr (MODE == MODE_FILTER || MODE == MODE_RETRY) named_sync(barid, 128);  // every append is in place
        if constexpr (MODE == MODE_BLOCK) {
            // nothing after the sweep: the chunk sums are the output
        } else if constexpr (MODE == MODE_SAMPLE) {
            // unused sample slots hold 0 (they rank below every valid sample)
            for (int it2 = n_tiles; it2 < SL_SAMPLE_TILES; ++it2)
                for (int qq = 0; qq < QH; ++qq) {
                    const int q = wg * QH + qq;
                    if (q < nq_here) a.samples[(row0 + q) * SL_SPR + it2 * SL_BN + et] = 0.f;
                }
            if (et < QH && wg * QH + et < nq_here) {
                // valid samples of the row: sampled keys j <= t - window
                const int q = wg * QH + et;
                const int64_t t = pos0 + q0 + q;
                // sampled keys S b <= t - window among the n_tiles * 128 read
                const int64_t lc = last_cand(p, t);
                const int64_t nv = lc >= 0 ? lc / S + 1 : 0;
                a.s_valid[row0 + q] = (int)min(nv, (int64_t)n_tiles * SL_BN);
            }
        } else if (ok) {
            // exact top-min(K, n) of every active row, ascending j, -1 padded
            for (int qq = kq; qq < QH; qq += 4) {
                const int q = wg * QH + qq;
                if (q >= nq_here) continue;
                const int64_t orow_off = ((int64_t)(b * p.hkv + g) * p.nq + a.i_begin + q0 + q) * p.topk;
                int32_t* orow = a.idx + orow_off;
                float* srow = a.sel_score ? a.sel_score + orow_off : nullptr;
                if (!r_act[q]) {
                    if (MODE == MODE_FILTER) {  // no candidates at all (t < window)
                        for (int u = lane; u < p.topk; u += 32) {
                            orow[u] = -1;
                            if (srow) srow[u] = -1.f;
                        }
                        if (lane == 0) a.status[row0 + q] = 0;
                    }
                    continue;
                }
                const int64_t t = pos0 + q0 + q;
                const int64_t n = last_cand(p, t) + 1;
                const int n_sel = (int)(n < p.topk ? n : p.topk);
                const int cnt = min(r_cnt[(L == ORDERED ? (n_tiles & 1) * QT : 0) + q], cmax);
                uint2* lst = lists + (int64_t)q * cmax;
                if (cnt < n_sel) {
                    if (lane == 0) a.status[row0 + q] = 1;  // the estimate was too high: retry
                    continue;
                }
                // the exact top n_sel (kth = 0 with every score >= 0 keeps them all)
                uint32_t kth = 0, jth = 0xffffffffu;
                if (cnt > n_sel) list_topk_bound(lst, cnt, (uint32_t)n_sel, hist + warp * 256, kth, jth);
                int written;
                if constexpr (L == ORDERED) {
                    written = warp_take(lst, cnt, kth, jth, orow, srow);  // the list is ascending in j
                } else if (n_sel <= SL_STAGE) {
                    // kept entries compacted in list order, their j staged over the dead Q
                    // tile and K ring (every MMA that read them has completed), then
                    // emitted ascending by j
                    int32_t* stage = reinterpret_cast<int32_t*>(sgen) + warp * SL_STAGE;
                    written = warp_compact(lst, cnt, kth, jth, stage);
                    warp_emit_sorted(lst, written, [&](int i) { return stage[i]; }, orow, srow);
                } else {
                    written = warp_compact(lst, cnt, kth, jth);
                    warp_emit_sorted(lst, written, [&](int i) { return (int32_t)lst[i].y; }, orow, srow);
                }
                __syncwarp();
                for (int u = written + lane; u < p.topk; u += 32) {
                    orow[u] = -1;
                    if (srow) srow[u] = -1.f;
                }
                // 0: selected by the filtered sweep; 2: selected by the retry pass (a
                // later call's filtered sweep overwrites every row's mark)
                if (lane == 0) a.status[row0 + q] = MODE == MODE_RETRY ? 2 : 0;
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Per row: tau = the r-th largest sample, r = ceil(L + 4.5 sqrt(L) + 2) with
// L = K s / n (s valid samples, n candidates); 0 when every candidate fits the
// survivor list, or when r exceeds s.
__global__ void __launch_bounds__(128) k2_thresh_kernel(Problem p, SelArgs a) {
    __shared__ uint32_t hist[4][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)p.B * p.hkv * a.i_count;
    const int64_t row = (int64_t)blockIdx.x * 4 + warp;
    if (row >= rows) return;
    const int qi = (int)(row % a.i_count);
    const int b = (int)(row / ((int64_t)p.hkv * a.i_count));
    const int64_t t = seq_pos0(p, b, KID_TOPK) + a.i_begin + qi;
    const int64_t n = last_cand(p, t) + 1;
    const int s = a.s_valid[row];
    float tau = 0.f;
    if (n > a.cmax / 2 && s > 0) {
        // L = samples expected above the K-th best candidate; the number that are
        // is about Poisson(L), so r = L + 4.5 sqrt(L) + 2 is reached with
        // probability about 1e-5 (the retry pass covers those rows), while about
        // r n / s candidates pass and the list compaction absorbs any overflow
        const float lam = (float)p.topk * (float)s / (float)n;
        int64_t r = (int64_t)ceilf(lam + 4.5f * sqrtf(lam) + 2.f);
        if (r <= s) {
            uint32_t kth, need_eq;
            warp_kth(reinterpret_cast<const uint32_t*>(a.samples + row * SL_SPR), 1, SL_SPR, (uint32_t)r, hist[warp],
                     kth, need_eq);
            tau = __uint_as_float(kth);
        }
    }
    if (lane == 0) a.tau[row] = tau;
}

// Block-level selection of one (query, group) row per warp from the chunk sums
// of the block sweep.  Block bb of size blk covers keys [bb blk, (bb + 1) blk);
// the candidate blocks are those lying wholly in [0, t - window], and the first
// keep = min(topk / blk, n_blk) of them in the order (score desc, bb asc) are
// kept, their keys written ascending, -1 padded to topk.  The warp first turns
// the row's chunk sums into block sums in place (block bb's chunks sit at or
// after position bb, so no unread chunk is overwritten), then runs the exact
// radix select on them.
__global__ void __launch_bounds__(128) k2_block_topk_kernel(Problem p, SelArgs a, int blk) {
    __shared__ uint32_t hist[4][256];
    __shared__ int32_t kept[4][64];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)p.B * p.hkv * a.i_count;
    const int64_t row = (int64_t)blockIdx.x * 4 + warp;
    if (row >= rows) return;
    const int qi = (int)(row % a.i_count);
    const int bg = (int)(row / a.i_count);  // b * H_kv + g
    const int b = bg / p.hkv;
    const int64_t t = seq_pos0(p, b, KID_TOPK) + a.i_begin + qi;
    const int64_t n_cand = last_cand(p, t) + 1 > 0 ? last_cand(p, t) + 1 : 0;
    const int n_blk = (int)(n_cand / blk);
    const int keep = min(p.topk / blk, n_blk);
    int32_t* orow = a.idx + ((int64_t)bg * p.nq + a.i_begin + qi) * p.topk;
    if (keep == n_blk || keep == 0) {  // every candidate block is kept (or none fits the budget)
        for (int u = lane; u < p.topk; u += 32) orow[u] = u < keep * blk ? u : -1;
        return;
    }
    float* cs = a.csum + row * a.cstride;
    const int nc = blk / 32;  // chunks per block
    if (nc > 1) {
        for (int base = 0; base < n_blk; base += 32) {
            const int bb = base + lane;
            float acc = 0.f;
            if (bb < n_blk)
                for (int c = 0; c < nc; ++c) acc += cs[(int64_t)bb * nc + c];
            __syncwarp();
            if (bb < n_blk) cs[bb] = acc;
            __syncwarp();
        }
    }
    uint32_t kth, need_eq;
    warp_kth(reinterpret_cast<const uint32_t*>(cs), 1, n_blk, (uint32_t)keep, hist[warp], kth, need_eq);
    // ordered keep: blocks above the k-th score plus the lowest-index equal ones
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t eq_seen = 0, written = 0;
    for (int base = 0; base < n_blk; base += 32) {
        const int bb = base + lane;
        const uint32_t x = bb < n_blk ? __float_as_uint(cs[bb]) : 0u;
        const bool eq = bb < n_blk && x == kth;
        const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
        const bool take = (bb < n_blk && x > kth) || (eq && eq_seen + __popc(eqb & lt) < need_eq);
        const uint32_t tb = __ballot_sync(0xffffffffu, take);
        if (take) kept[warp][written + __popc(tb & lt)] = bb;
        eq_seen += __popc(eqb);
        written += __popc(tb);
    }
    __syncwarp();
    for (int u = lane; u < p.topk; u += 32) {
        const int i = u / blk;
        orow[u] = i < keep ? kept[warp][i] * blk + (u - i * blk) : -1;
    }
}

// [B][H_q][n_q][D] bf16 seen as (D, H_q, n_q, B) with box (64, G, qt, 1): the
// shared-memory tile rows come out ordered (query, head), 128 bytes each.
bool make_q_map(CUtensorMap* m, const void* base, int D, int hq, int nq, int B, int G, int qt) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)hq, (cuuint64_t)nq, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)nq * D * 2, (cuuint64_t)D * 2, (cuuint64_t)hq * nq * D * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)qt, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, int G, int MODE, int L>
cudaError_t launch_mode(const Problem& p, const CUtensorMap& mq, const CUtensorMap& mk, const SelArgs& a,
                        cudaStream_t st) {
    using C = SlCfg<D, G, L>;
    auto kern = k2_select_tc_kernel<D, G, MODE, L>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid((a.i_count + C::QT - 1) / C::QT, p.hkv, p.B);
    prof_begin(MODE == MODE_SAMPLE   ? KID_SCORE
               : MODE == MODE_FILTER ? KID_FILTER
               : MODE == MODE_RETRY  ? KID_RETRY
                                     : KID_BLOCK_SWEEP,
               st);
    kern<<<grid, C::THREADS, C::SMEM, st>>>(mq, mk, p, a);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

// K seen with rows S apart: (D, kv_len / S, B * H_kv), box (64, 128, 1).
bool make_strided_map(CUtensorMap* m, const void* base, int D, int64_t kv_len, int64_t S, int64_t z) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)(kv_len / S), (cuuint64_t)z};
    cuuint64_t strides[2] = {(cuuint64_t)(S * D * 2), (cuuint64_t)(kv_len * D * 2)};
    cuuint32_t box[3] = {64, (cuuint32_t)SL_BN, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, int G, int L>
cudaError_t launch_select_dgl(const Problem& p, const void* q, const void* k, const SelArgs& a, cudaStream_t st) {
    CUtensorMap mq, mk, mks;
    if (!make_q_map(&mq, q, D, p.hq, p.nq, p.B, G, Lay<L>::QT) ||
        !make_map(&mk, k, D, (uint64_t)p.kv_len, (uint64_t)p.B * p.hkv, 128) ||
        !make_strided_map(&mks, k, D, p.kv_len, a.sample_stride, (int64_t)p.B * p.hkv))
        return cudaErrorInvalidValue;
    cudaError_t e = launch_mode<D, G, MODE_SAMPLE, L>(p, mq, mks, a, st);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)p.B * p.hkv * a.i_count;
    prof_begin(KID_THRESH, st);
    k2_thresh_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(p, a);
    prof_end(st);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_mode<D, G, MODE_FILTER, L>(p, mq, mk, a, st)) != cudaSuccess) return e;
    return launch_mode<D, G, MODE_RETRY, L>(p, mq, mk, a, st);
}

template <int D, int G>
cudaError_t launch_select_dg(const Problem& p, const void* q, const void* k, const SelArgs& a, int layout,
                             cudaStream_t st) {
    if constexpr (kCounterFits<G>) {
        if (layout == COUNTER) return launch_select_dgl<D, G, COUNTER>(p, q, k, a, st);
    }
    return launch_select_dgl<D, G, ORDERED>(p, q, k, a, st);
}

template <int D, int G, int L>
cudaError_t launch_block_dgl(const Problem& p, const void* q, const void* k, const SelArgs& a, cudaStream_t st) {
    CUtensorMap mq, mk;
    if (!make_q_map(&mq, q, D, p.hq, p.nq, p.B, G, Lay<L>::QT) ||
        !make_map(&mk, k, D, (uint64_t)p.kv_len, (uint64_t)p.B * p.hkv, 128))
        return cudaErrorInvalidValue;
    return launch_mode<D, G, MODE_BLOCK, L>(p, mq, mk, a, st);
}

template <int D, int G>
cudaError_t launch_block_dg(const Problem& p, const void* q, const void* k, const SelArgs& a, int layout,
                            cudaStream_t st) {
    if constexpr (kCounterFits<G>) {
        if (layout == COUNTER) return launch_block_dgl<D, G, COUNTER>(p, q, k, a, st);
    }
    return launch_block_dgl<D, G, ORDERED>(p, q, k, a, st);
}

template <int D>
cudaError_t launch_block_d(const Problem& p, const void* q, const void* k, const SelArgs& a, int layout,
                           cudaStream_t st) {
    switch (p.hq / p.hkv) {
        case 1: return launch_block_dg<D, 1>(p, q, k, a, layout, st);
        case 2: return launch_block_dg<D, 2>(p, q, k, a, layout, st);
        case 4: return launch_block_dg<D, 4>(p, q, k, a, layout, st);
        default: return launch_block_dg<D, 8>(p, q, k, a, layout, st);
    }
}

template <int D>
cudaError_t launch_select_d(const Problem& p, const void* q, const void* k, const SelArgs& a, int layout,
                            cudaStream_t st) {
    switch (p.hq / p.hkv) {
        case 1: return launch_select_dg<D, 1>(p, q, k, a, layout, st);
        case 2: return launch_select_dg<D, 2>(p, q, k, a, layout, st);
        case 4: return launch_select_dg<D, 4>(p, q, k, a, layout, st);
        default: return launch_select_dg<D, 8>(p, q, k, a, layout, st);
    }
}

}  // namespace

// The epilogue layout of a call whose longest row has n_cand_max candidates.
static int select_tc_layout(int64_t n_cand_max, int G) {
    const bool fits = G == 4 ? kCounterFits<4> : G == 8 ? kCounterFits<8> : false;
    return n_cand_max >= SL_COUNTER_MIN_CAND && fits ? COUNTER : ORDERED;
}

int select_tc_qt(int64_t n_cand_max, int G) {
    return select_tc_layout(n_cand_max, G) == COUNTER ? Lay<COUNTER>::QT : Lay<ORDERED>::QT;
}

// Layout, survivor list capacity and slot count of a call over queries with up
// to n_cand_max candidates, in CTAs of the layout's qt queries.
static void select_tc_geometry(const Problem& p, int i_count, int64_t n_cand_max, int& layout, int& qt, int& cmax,
                               int& n_slots, int& by_block) {
    layout = select_tc_layout(n_cand_max, p.hq / p.hkv);
    qt = layout == COUNTER ? Lay<COUNTER>::QT : Lay<ORDERED>::QT;
    cmax = n_cand_max <= SL_CMAX ? (int)((n_cand_max + 31) / 32 * 32) : SL_CMAX;
    if (cmax < 32) cmax = 32;
    const int64_t grid = (int64_t)((i_count + qt - 1) / qt) * p.hkv * p.B;
    by_block = grid <= SL_SLOTS;
    n_slots = by_block ? (int)grid : SL_SLOTS;
}

size_t select_tc_scratch_bytes(const Problem& p, int i_count, int64_t n_cand_max) {
    int layout, qt, cmax, n_slots, by_block;
    select_tc_geometry(p, i_count, n_cand_max, layout, qt, cmax, n_slots, by_block);
    const int64_t rows = (int64_t)p.B * p.hkv * i_count;
    const size_t per_row = SL_SPR * 4 + 3 * 4;
    return (size_t)n_slots * qt * cmax * sizeof(uint2) + (size_t)rows * per_row;
}

size_t select_tc_status_offset(const Problem& p, int i_count, int64_t n_cand_max) {
    int layout, qt, cmax, n_slots, by_block;
    select_tc_geometry(p, i_count, n_cand_max, layout, qt, cmax, n_slots, by_block);
    const int64_t rows = (int64_t)p.B * p.hkv * i_count;
    return (size_t)n_slots * qt * cmax * sizeof(uint2) + (size_t)rows * (SL_SPR * 4 + 2 * 4);
}

cudaError_t launch_select_tc(const Problem& p, const void* q, const void* k, const float* lse, int32_t* idx,
                             void* scratch, int i_begin, int i_count, int64_t n_cand_max, cudaStream_t st,
                             float* sel_score) {
    const int64_t rows = (int64_t)p.B * p.hkv * i_count;
    uint8_t* base = reinterpret_cast<uint8_t*>(scratch);
    SelArgs a{};
    int layout, qt, n_slots;
    select_tc_geometry(p, i_count, n_cand_max, layout, qt, a.cmax, n_slots, a.slot_by_block);
    a.sample_stride = p.kv_len / (SL_SAMPLE_TILES * SL_BN) > 1 ? p.kv_len / (SL_SAMPLE_TILES * SL_BN) : 1;
    a.lse = lse;
    a.idx = idx;
    a.sel_score = sel_score;
    a.slots = reinterpret_cast<uint2*>(base);
    base += (size_t)n_slots * qt * a.cmax * sizeof(uint2);
    a.samples = reinterpret_cast<float*>(base);
    base += (size_t)rows * SL_SPR * 4;
    a.s_valid = reinterpret_cast<int32_t*>(base);
    base += (size_t)rows * 4;
    a.tau = reinterpret_cast<float*>(base);
    base += (size_t)rows * 4;
    a.status = reinterpret_cast<int32_t*>(base);
    a.i_begin = i_begin;
    a.i_count = i_count;
    if (p.D == 64) return launch_select_d<64>(p, q, k, a, layout, st);
    return launch_select_d<128>(p, q, k, a, layout, st);
}

// Chunk sums: one float per 32 keys of every candidate tile, rows of cstride.
static int64_t block_cstride(int64_t n_cand_max) { return (n_cand_max + SL_BN - 1) / SL_BN * (SL_BN / 32); }

size_t block_tc_scratch_bytes(const Problem& p, int i_count, int64_t n_cand_max) {
    if (n_cand_max <= 0) return 0;
    return (size_t)p.B * p.hkv * i_count * block_cstride(n_cand_max) * 4;
}

cudaError_t launch_block_select_tc(const Problem& p, const void* q, const void* k, const float* lse, int32_t* idx,
                                   void* scratch, int i_begin, int i_count, int64_t n_cand_max, int blk,
                                   cudaStream_t st) {
    SelArgs a{};
    a.lse = lse;
    a.idx = idx;
    a.i_begin = i_begin;
    a.i_count = i_count;
    a.csum = reinterpret_cast<float*>(scratch);
    a.cstride = block_cstride(n_cand_max);
    // the sweep only runs when some row has more candidate blocks than the budget
    if (n_cand_max / blk > p.topk / blk && p.topk >= blk) {
        // the token sweep's epilogue geometry for this candidate count (the chunk
        // sums are the same in both)
        const int layout = select_tc_layout(n_cand_max, p.hq / p.hkv);
        const cudaError_t e = p.D == 64 ? launch_block_d<64>(p, q, k, a, layout, st)
                                        : launch_block_d<128>(p, q, k, a, layout, st);
        if (e != cudaSuccess) return e;
    }
    const int64_t rows = (int64_t)p.B * p.hkv * i_count;
    prof_begin(KID_BLOCK_TOPK, st);
    k2_block_topk_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(p, a, blk);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

}  // namespace hs2
