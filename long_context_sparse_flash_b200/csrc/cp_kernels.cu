// cp_kernels.cu -- the merge steps of context parallelism: the KV cache of one
// long context is cut into P contiguous slices, one per GPU; every rank runs
// the full layer, the selection and the sparse layers over its own slice, and
// these kernels turn the P per-slice results into the exact single-cache ones:
//
//   cp_combine_kernel      P partial attention results (output, natural-log LSE
//                          over the slice's keys) -> the attention over the union
//                          of the keys:  lse = ln sum_p e^(lse_p),
//                          out = sum_p e^(lse_p - lse) out_p
//   cp_select_merge_kernel P per-slice top-K lists (local rows and scores, each
//                          ascending) -> the exact top-K over the whole context:
//                          the global top-K is contained in the union of the
//                          per-slice top-Ks, slices are contiguous and in order,
//                          so the concatenated lists are ascending in j and the
//                          usual select (ties to the lower j) applies
//   cp_idx_local_kernel    a whole-context selection -> the rows one slice holds,
//                          shifted to the slice's local row numbers
//
// The scores are the group-summed probabilities normalised with the GLOBAL LSE
// (the slices' selection passes read the combined LSE), so they compare across
// slices.  HySparse2 pages: xiawanshe.com report, section "两级KV共享" (one full
// layer, its KV cache and selection reused by the sparse layers) and section
// "Token级选择" (per-token selection over the whole older context).
#include "hs2_kernels.h"

namespace hs2 {

namespace {

// One warp per row (sequence, head, query).
template <int D>
__global__ void __launch_bounds__(256) cp_combine_kernel(int n_parts, int64_t rows,
                                                         const __nv_bfloat16* __restrict__ out_parts,
                                                         const float* __restrict__ lse_parts,
                                                         __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    constexpr int E = D / 32;  // elements per lane
    float M = -INFINITY;
    for (int s = 0; s < n_parts; ++s) M = fmaxf(M, lse_parts[(int64_t)s * rows + row]);
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    float L = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < n_parts; ++s) {
            const float ls = lse_parts[(int64_t)s * rows + row];
            const float w = ls == -INFINITY ? 0.f : ex2((ls - M) * kLog2e);
            L += w;
            const __nv_bfloat16* o = out_parts + ((int64_t)s * rows + row) * D + lane * E;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += w * __bfloat162float(o[e]);
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16* orow = out + row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) *reinterpret_cast<uint32_t*>(orow + e) = pack_bf16(acc[e] * inv, acc[e + 1] * inv);
    if (lane == 0) lse[row] = L > 0.f ? M + __logf(L) : -INFINITY;
}

constexpr int CP_MAX_PARTS = 16;

struct MergeArgs {
    int n_parts;
    int64_t rows;                     // B * H_kv * n_q
    int topk;
    const int32_t* idx_parts;         // [P][rows][topk] local rows, ascending, -1 padded
    const float* score_parts;         // [P][rows][topk]
    int64_t off[CP_MAX_PARTS];        // first key of each slice (ascending)
    int32_t* idx;                     // [rows][topk] whole-context rows
};

// One warp per (sequence, group, query) row.  The row's candidate lists are
// the valid prefixes of the P parts; an 8-bit radix select over their fp32
// score bits finds the k-th score, then one ordered pass keeps the entries
// above it and the first ones equal to it.
__global__ void __launch_bounds__(128) cp_select_merge_kernel(MergeArgs a) {
    __shared__ uint32_t hist_s[4][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 4 + warp;
    if (row >= a.rows) return;
    uint32_t* hist = hist_s[warp];
    const int K = a.topk;
    int32_t* orow = a.idx + row * K;
    // valid entries of each part (a prefix)
    int cnt[CP_MAX_PARTS];
    int total = 0;
    for (int s = 0; s < a.n_parts; ++s) {
        const int32_t* ir = a.idx_parts + ((int64_t)s * a.rows + row) * K;
        int c = 0;
        for (int u = lane; u < K; u += 32) c += ir[u] >= 0;
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        cnt[s] = c;
        total += c;
    }
    const int n_sel = total < K ? total : K;
    uint32_t kth = 0u, need_eq = 0xffffffffu;  // total <= K: every entry is kept
    if (total > K) {
        uint32_t prefix = 0, pmask = 0, k_rem = (uint32_t)K;
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int u = lane; u < 256; u += 32) hist[u] = 0;
            __syncwarp();
            for (int s = 0; s < a.n_parts; ++s) {
                const uint32_t* sr =
                    reinterpret_cast<const uint32_t*>(a.score_parts + ((int64_t)s * a.rows + row) * K);
                for (int u = lane; u < cnt[s]; u += 32) {
                    const uint32_t x = sr[u];
                    if ((x & pmask) == prefix) atomicAdd(&hist[(x >> shift) & 255u], 1u);
                }
            }
            __syncwarp();
            // lane l owns digits 8 (31 - l) .. + 7, so lane order is descending digit
            uint32_t bins[8], sum = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                bins[u] = hist[8 * (31 - lane) + u];
                sum += bins[u];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const uint32_t excl = incl - sum;
            const bool mine = excl < k_rem && k_rem <= incl;
            uint32_t digit = 0, krem_new = 0;
            if (mine) {
                uint32_t above = excl;
#pragma unroll
                for (int u = 7; u >= 0; --u) {
                    if (above + bins[u] >= k_rem) {
                        digit = 8 * (31 - lane) + u;
                        krem_new = k_rem - above;
                        break;
                    }
                    above += bins[u];
                }
            }
            const uint32_t who = __ballot_sync(0xffffffffu, mine);
            const int src = who ? __ffs(who) - 1 : 0;
            digit = __shfl_sync(0xffffffffu, digit, src);
            krem_new = __shfl_sync(0xffffffffu, krem_new, src);
            prefix |= digit << shift;
            pmask |= 255u << shift;
            k_rem = krem_new;
            __syncwarp();
        }
        kth = prefix;
        need_eq = k_rem;
    }
    // ordered keep over the parts in slice order (ascending whole-context rows)
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t eq_seen = 0, written = 0;
    for (int s = 0; s < a.n_parts; ++s) {
        const int32_t* ir = a.idx_parts + ((int64_t)s * a.rows + row) * K;
        const uint32_t* sr = reinterpret_cast<const uint32_t*>(a.score_parts + ((int64_t)s * a.rows + row) * K);
        for (int base = 0; base < cnt[s]; base += 32) {
            const int u = base + lane;
            const bool valid = u < cnt[s];
            const uint32_t x = valid ? sr[u] : 0u;
            const bool eq = valid && x == kth;
            const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
            const bool take = (valid && (total <= K || x > kth)) ||
                              (total > K && eq && eq_seen + __popc(eqb & lt) < need_eq);
            const uint32_t tb = __ballot_sync(0xffffffffu, take);
            if (take) orow[written + __popc(tb & lt)] = (int32_t)(ir[u] + a.off[s]);
            eq_seen += __popc(eqb);
            written += __popc(tb);
        }
    }
    for (int u = n_sel + lane; u < K; u += 32) orow[u] = -1;
}

// One warp per (sequence, group, query) row: keep the entries in [off, off + len),
// shifted by -off, in order; -1 after them.
__global__ void __launch_bounds__(128) cp_idx_local_kernel(int64_t rows, int topk, const int32_t* __restrict__ idx,
                                                           int64_t off, int64_t len, int32_t* __restrict__ out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 4 + warp;
    if (row >= rows) return;
    const int32_t* ir = idx + row * topk;
    int32_t* orow = out + row * topk;
    const uint32_t lt = (1u << lane) - 1u;
    int written = 0;
    for (int base = 0; base < topk; base += 32) {
        const int u = base + lane;
        const int64_t j = u < topk ? (int64_t)ir[u] : -1;
        const bool mine = j >= off && j < off + len;
        const uint32_t b = __ballot_sync(0xffffffffu, mine);
        if (mine) orow[written + __popc(b & lt)] = (int32_t)(j - off);
        written += __popc(b);
    }
    for (int u = written + lane; u < topk; u += 32) orow[u] = -1;
}

}  // namespace

cudaError_t launch_cp_combine(int n_parts, int64_t rows, int head_dim, const void* out_parts, const float* lse_parts,
                              void* out, float* lse, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows * 32 + 255) / 256);
    prof_begin(KID_CP_COMBINE, st);
    if (head_dim == 64)
        cp_combine_kernel<64><<<grid, 256, 0, st>>>(n_parts, rows, (const __nv_bfloat16*)out_parts, lse_parts,
                                                     (__nv_bfloat16*)out, lse);
    else
        cp_combine_kernel<128><<<grid, 256, 0, st>>>(n_parts, rows, (const __nv_bfloat16*)out_parts, lse_parts,
                                                      (__nv_bfloat16*)out, lse);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

int cp_max_parts() { return CP_MAX_PARTS; }

cudaError_t launch_cp_select_merge(int n_parts, int64_t rows, int topk, const int32_t* idx_parts,
                                   const float* score_parts, const int64_t* offs, int32_t* idx, cudaStream_t st) {
    if (rows == 0 || topk == 0) return cudaSuccess;
    MergeArgs a{};
    a.n_parts = n_parts;
    a.rows = rows;
    a.topk = topk;
    a.idx_parts = idx_parts;
    a.score_parts = score_parts;
    for (int s = 0; s < n_parts; ++s) a.off[s] = offs[s];
    a.idx = idx;
    prof_begin(KID_CP_MERGE, st);
    cp_select_merge_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(a);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_cp_idx_local(int64_t rows, int topk, const int32_t* idx, int64_t off, int64_t len, int32_t* out,
                                cudaStream_t st) {
    if (rows == 0 || topk == 0) return cudaSuccess;
    prof_begin(KID_CP_IDX, st);
    cp_idx_local_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(rows, topk, idx, off, len, out);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

}  // namespace hs2
