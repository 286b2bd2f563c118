// k3_sparse_attn.cu -- K3: one sparse KV-reuse layer of HySparse2's
// Cross-Decoder (xiawanshe.com report, section "两级KV共享": the following
// sparse layers reuse the full layer's cache and token selection; section
// "Token级选择": each attends to the selected older tokens plus the forced
// most-recent window, all from the one shared cache).
//
// One CTA = one (sequence, query, KV group); its G heads share every gathered
// K/V row.  The attended rows S = idx U window (the selection's valid prefix,
// then the window) are cut into 16-row tiles and gathered with 16-byte
// cp.async into a ring of SP_STAGES swizzled stages; each tile's row indices
// are fetched into registers a tile before its copies are issued, so shared
// memory holds only the staging.  One warp per CTA: the gather is
// latency-bound, and many small CTAs per SM keep the most tiles in flight.
// Per tile:
//   S^T (16 keys x 8 heads) = K_tile Q^T      mma.sync m16n8k16, A = K rows
//   P^T = 2^(S^T - m) per head column, online softmax over the warp's tiles
//   O^T (D x 8 heads) += V_tile^T P^T         A = V^T via ldmatrix.trans,
//                                             B = P^T via movmatrix.trans
// The group's heads sit in the MMA's N = 8 columns (padded when G < 8), so no
// tensor-core work is spent on padding rows of M.  With W > 1 warps per CTA the
// warps' partial (max, sum, O) are merged exactly at the end.
//
// Two further uses share the kernel: with_window = 0 attends to the selected
// rows alone (the selected branch of the predecessor design's two-branch layer),
// and a non-null lse receives the natural-log LSE of the attended logits (both
// branches, and the per-slice partials of context parallelism, are merged by
// it).  A query with no attended row writes 0 and LSE -inf.
#include "hs2_kernels.h"

namespace hs2 {

namespace {

// One warp per CTA when the grid fills the machine (more, smaller CTAs per SM
// hide the gather latency best); four when it does not (decode-sized calls),
// each warp then taking every fourth tile of the row.
constexpr int SP_SMALL_GRID = 4 * 148;
constexpr int SP_STAGES = 2;  // tiles in the staging ring

template <int D, int W>
struct K3Cfg {
    static constexpr int CH = D / 8;
    static constexpr int TILE_BYTES = 16 * D * 2;                 // one 16-row K (or V) tile
    static constexpr int WARP_BYTES = SP_STAGES * 2 * TILE_BYTES;  // stages x (K, V)
    static constexpr int STAGE_BYTES = W * WARP_BYTES;
    static constexpr int COMB_BYTES = W * (D * 8 + 16) * 4;  // per warp: O^T, m, l
    static constexpr int FIXED = STAGE_BYTES > COMB_BYTES ? STAGE_BYTES : COMB_BYTES;
};

template <int D, int G, int W>
__global__ void __launch_bounds__(W * 32) k3_sparse_kernel(Problem p, const __nv_bfloat16* __restrict__ q,
                                                                   const __nv_bfloat16* __restrict__ k,
                                                                   const __nv_bfloat16* __restrict__ v,
                                                                   const int32_t* __restrict__ idx,
                                                                   __nv_bfloat16* __restrict__ out,
                                                                   int with_window, float* __restrict__ lse) {
    using C = K3Cfg<D, W>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int64_t pos0 = seq_pos0(p, b, KID_SPARSE);
    const int64_t t = pos0 + i;
    const int64_t w0 = t - p.window + 1 > 0 ? t - p.window + 1 : 0;
    // last window key held by the buffer (a slice of a longer context may end
    // before t, or start after it: then fewer or no window rows are here)
    const int64_t w_hi = min(t, p.kv_len - 1);
    const int nwin = (with_window && w_hi >= w0) ? (int)(w_hi - w0 + 1) : 0;  // 0: the selected rows alone

    // attended rows: the selection's valid prefix (its length counted here),
    // then the window
    const int32_t* irow = idx + ((int64_t)(b * p.hkv + g) * p.nq + i) * p.topk;
    int cnt = 0;
    for (int r = lane; r < p.topk; r += 32) {
        const int32_t j = irow[r];
        cnt += j >= 0;
#ifdef HS2_CHECKED
        const bool bad_range = j < -1 || (int64_t)j > t - p.window;
        const bool bad_order = r > 0 && j >= 0 && (irow[r - 1] < 0 || irow[r - 1] >= j);
        if (bad_range || bad_order) report_error(p.err, HS2_ERR_DEVICE_CHECK, KID_SPARSE, (uint32_t)i, (uint32_t)r);
#endif
    }
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 16);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 8);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 4);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 2);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 1);
    const int nsel = cnt;
    const int n = nsel + nwin;
    const int n_mt = (n + 15) / 16;
    // row index of attended position li, -1 past the end or when invalid
    auto row_of = [&](int li) -> int32_t {
        int32_t j = -1;
        if (li < nsel)
            j = irow[li];
        else if (li < n)
            j = (int32_t)(w0 + (li - nsel));
        return (j >= 0 && (int64_t)j <= t) ? j : -1;
    };

    // Q^T B fragments: column = head (lane / 4) of the group, zero beyond G
    uint32_t qb[D / 16][2];
    {
        const int hh = lane >> 2;
        const bool ok = hh < G;
        const __nv_bfloat16* qrow = q + ((int64_t)(b * p.hq + g * G + (ok ? hh : 0)) * p.nq + i) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int d0 = ks * 16 + 2 * (lane & 3);
            qb[ks][0] = ok ? *reinterpret_cast<const uint32_t*>(qrow + d0) : 0u;
            qb[ks][1] = ok ? *reinterpret_cast<const uint32_t*>(qrow + d0 + 8) : 0u;
        }
    }

    const __nv_bfloat16* kg = k + ((int64_t)(b * p.hkv + g) * p.kv_len) * D;
    const __nv_bfloat16* vg = v + ((int64_t)(b * p.hkv + g) * p.kv_len) * D;
    const uint32_t s_w = smem_u32(smem) + warp * C::WARP_BYTES;
    // Tile loads: lanes 0-15 copy one row and lanes 16-31 the next (16-byte
    // chunk = lane % 16 for D = 128), eight row pairs per 16-row tile.  Lane l
    // holds the index of the tile's row l % 16 and the others take it by shuffle;
    // the swizzled chunk is (lane chunk ^ row parity) ^ (2 * it mod 8).
    auto load_tile = [&](int stage, int32_t myj) {
        const uint32_t sk = s_w + stage * 2 * C::TILE_BYTES;
        constexpr int RPI = 32 / C::CH;  // rows per iteration (2 for D = 128, 4 for D = 64)
        const int hi = lane / C::CH, ch = lane % C::CH;
#pragma unroll
        for (int it = 0; it < 16 / RPI; ++it) {
            const int r = it * RPI + hi;
            const int32_t j = __shfl_sync(0xffffffffu, myj, r);
            const size_t goff = (size_t)(j < 0 ? 0 : j) * (size_t)(D * 2) + (size_t)ch * 16u;
            const uint32_t so = sk + swz<C::CH>(r, ch);
            cp_async16(so, (const char*)kg + goff, j < 0 ? 0 : 16);
            cp_async16(so + C::TILE_BYTES, (const char*)vg + goff, j < 0 ? 0 : 16);
        }
    };

    float acc[D / 16][4];
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) acc[dt][0] = acc[dt][1] = acc[dt][2] = acc[dt][3] = 0.f;
    float m_c[2] = {-INFINITY, -INFINITY}, l_c[2] = {0.f, 0.f};

    // This warp's tiles are warp, warp + W, ...: its k-th tile lives in stage
    // k % SP_STAGES; tiles k + 1 .. k + SP_STAGES - 1 are in flight while tile k is
    // computed.  jr[u] = row index of its tile k + u (lane l: row l % 16), u <
    // SP_STAGES; the next one is fetched a tile ahead.
    const int r16 = lane & 15;
    const int n_loc = warp < n_mt ? (n_mt - warp + W - 1) / W : 0;
    auto tile_row = [&](int kk) { return (warp + kk * W) * 16 + r16; };
    int32_t jr[SP_STAGES];
#pragma unroll
    for (int u = 0; u < SP_STAGES; ++u) jr[u] = row_of(tile_row(u));
#pragma unroll
    for (int u = 0; u < SP_STAGES - 1; ++u) {
        if (u < n_loc) load_tile(u, jr[u]);
        cp_async_commit();
    }
    int stage = 0;
    for (int kt = 0; kt < n_loc; ++kt) {
        const int32_t j_next = row_of(tile_row(kt + SP_STAGES));
        const int lstage = (stage + SP_STAGES - 1) % SP_STAGES;
        if (kt + SP_STAGES - 1 < n_loc) load_tile(lstage, jr[SP_STAGES - 1]);
        cp_async_commit();
        cp_async_wait<SP_STAGES - 1>();
        __syncwarp();
        const uint32_t sk = s_w + stage * 2 * C::TILE_BYTES, sv = sk + C::TILE_BYTES;

        // two independent accumulation chains (even / odd k-steps) halve the MMA latency
        float c[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a[4];
            const int mi = lane >> 3;
            ldsm_x4(a, sk + swz<C::CH>((mi & 1) * 8 + (lane & 7), 2 * ks + (mi >> 1)));
            mma16816((ks & 1) ? c2 : c, a, qb[ks]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) c[e] += c2[e];
        // rows lane/4 and lane/4 + 8 of the tile; columns 2*(lane%4) + {0, 1}
        bool row_ok[2];
        row_ok[0] = __shfl_sync(0xffffffffu, jr[0], lane >> 2) >= 0;
        row_ok[1] = __shfl_sync(0xffffffffu, jr[0], (lane >> 2) + 8) >= 0;
        float s[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) s[e] = row_ok[e >> 1] ? c[e] * p.scale_log2 : -INFINITY;
        float alpha[2], m_use[2];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            float mx = fmaxf(s[cc], s[cc + 2]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m_c[cc], mx);
            m_use[cc] = m_new == -INFINITY ? 0.f : m_new;
            alpha[cc] = ex2(m_c[cc] - m_use[cc]);
            m_c[cc] = m_new;
            l_c[cc] *= alpha[cc];
        }
        float pr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            pr[e] = ex2(s[e] - m_use[e & 1]);
            l_c[e & 1] += pr[e];
        }
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt) {
            acc[dt][0] *= alpha[0];
            acc[dt][1] *= alpha[1];
            acc[dt][2] *= alpha[0];
            acc[dt][3] *= alpha[1];
        }
        uint32_t pb[2];
        pb[0] = movm_t(pack_bf16(pr[0], pr[1]));
        pb[1] = movm_t(pack_bf16(pr[2], pr[3]));
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt) {
            uint32_t a[4];
            const int mi = lane >> 3;
            ldsm_x4_t(a, sv + swz<C::CH>((mi >> 1) * 8 + (lane & 7), 2 * dt + (mi & 1)));
            mma16816(acc[dt], a, pb);
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u + 1 < SP_STAGES; ++u) jr[u] = jr[u + 1];
        jr[SP_STAGES - 1] = j_next;
        stage = stage + 1 == SP_STAGES ? 0 : stage + 1;
    }
    cp_async_wait<0>();

    // per-warp column sums, then the exact merge of the warps' partial states
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        l_c[cc] += __shfl_xor_sync(0xffffffffu, l_c[cc], 4);
        l_c[cc] += __shfl_xor_sync(0xffffffffu, l_c[cc], 8);
        l_c[cc] += __shfl_xor_sync(0xffffffffu, l_c[cc], 16);
    }
    __syncthreads();  // staging is reused for the merge
    float* comb = reinterpret_cast<float*>(smem);
    float* ot = comb + warp * (D * 8 + 16);  // [D][8] then m[8], l[8]
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int d = dt * 16 + (lane >> 2) + 8 * (e >> 1);
            const int col = 2 * (lane & 3) + (e & 1);
            ot[d * 8 + col] = acc[dt][e];
        }
    }
    if ((lane >> 2) == 0) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            ot[D * 8 + 2 * lane + cc] = m_c[cc];
            ot[D * 8 + 8 + 2 * lane + cc] = l_c[cc];
        }
    }
    __syncthreads();
    for (int u = tid; u < G * D; u += W * 32) {
        const int hh = u / D, d = u % D;
        float mm = -INFINITY;
#pragma unroll
        for (int w = 0; w < W; ++w) mm = fmaxf(mm, comb[w * (D * 8 + 16) + D * 8 + hh]);
        float num = 0.f, den = 0.f;
        if (mm != -INFINITY) {  // else no attended row at all (the selected rows alone, none valid)
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const float* wb = comb + w * (D * 8 + 16);
                const float sc = ex2(wb[D * 8 + hh] - mm);
                num += sc * wb[d * 8 + hh];
                den += sc * wb[D * 8 + 8 + hh];
            }
        }
        const int64_t oh = (int64_t)(b * p.hq + g * G + hh) * p.nq + i;
        out[oh * D + d] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
        // natural-log LSE of the attended logits: (m + log2 l) ln 2 in the kernel's log2 units
        if (lse != nullptr && d == 0) lse[oh] = den > 0.f ? (mm + __log2f(den)) * kLn2 : -INFINITY;
    }
}

template <int D, int G, int W>
cudaError_t launch_sparse_dgw(const Problem& p, const void* q, const void* k, const void* v, const int32_t* idx,
                              void* out, int with_window, float* lse, cudaStream_t st) {
    using C = K3Cfg<D, W>;
    const int smem = C::FIXED;
    auto kern = k3_sparse_kernel<D, G, W>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.nq, p.hkv, p.B);
    prof_begin(KID_SPARSE, st);
    kern<<<grid, W * 32, smem, st>>>(p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                     idx, (__nv_bfloat16*)out, with_window, lse);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_sparse_dg(const Problem& p, const void* q, const void* k, const void* v, const int32_t* idx,
                             void* out, int with_window, float* lse, cudaStream_t st) {
    const int64_t ctas = (int64_t)p.nq * p.hkv * p.B;
    if (ctas < SP_SMALL_GRID) return launch_sparse_dgw<D, G, 4>(p, q, k, v, idx, out, with_window, lse, st);
    return launch_sparse_dgw<D, G, 1>(p, q, k, v, idx, out, with_window, lse, st);
}

template <int D>
cudaError_t launch_sparse_d(const Problem& p, const void* q, const void* k, const void* v, const int32_t* idx,
                            void* out, int with_window, float* lse, cudaStream_t st) {
    switch (p.hq / p.hkv) {
        case 1: return launch_sparse_dg<D, 1>(p, q, k, v, idx, out, with_window, lse, st);
        case 2: return launch_sparse_dg<D, 2>(p, q, k, v, idx, out, with_window, lse, st);
        case 4: return launch_sparse_dg<D, 4>(p, q, k, v, idx, out, with_window, lse, st);
        default: return launch_sparse_dg<D, 8>(p, q, k, v, idx, out, with_window, lse, st);
    }
}

}  // namespace

cudaError_t launch_sparse(const Problem& p, const void* q, const void* k, const void* v, const int32_t* idx,
                          void* out, cudaStream_t st, int with_window, float* lse) {
    if (p.D == 64) return launch_sparse_d<64>(p, q, k, v, idx, out, with_window, lse, st);
    return launch_sparse_d<128>(p, q, k, v, idx, out, with_window, lse, st);
}

}  // namespace hs2
