// k1_decode.cu -- decode step of the Cross-Decoder's full-attention layer with
// token selection (HySparse2; xiawanshe.com report, sections "两级KV共享" and
// "Token级选择"): one new token per sequence attends to its whole cache and
// picks its top-K older tokens.
//
// With one query per sequence the work is a stream over the cache, so it is
// split over many CTAs:
//   k1d_partial_kernel  one CTA per (sequence, KV group, chunk of keys): the
//       G heads' partial online-softmax state (max, sum, O) over the chunk, and
//       the scaled logits s2_{h,j} of every candidate key (j <= t - window),
//       stored [group][j][head] so the selection never re-reads K.
//       S^T = K Q^T and O^T += V^T P^T on mma.sync m16n8k16 (the group's heads
//       in N), K/V rows staged by cp.async in a per-warp ring.
//   k1d_combine_kernel  exact merge of the chunks' states -> out, lse.
//   k2d_score_kernel    score_j = sum_h 2^(s2_{h,j} - lse2_h) from the stored
//       logits; the exact radix top-k kernel then selects over the scores.
#include "hs2_kernels.h"

namespace hs2 {

namespace {

constexpr int DC_WARPS = 4;
constexpr int DC_NST = 3;  // per-warp ring stages

template <int D>
struct DcCfg {
    static constexpr int CH = D / 8;
    static constexpr int TILE = 16 * D * 2;            // 16 rows of K (or V)
    static constexpr int WARP_BYTES = DC_NST * 2 * TILE;
    static constexpr int STAGE_BYTES = DC_WARPS * WARP_BYTES;
    static constexpr int COMB_BYTES = DC_WARPS * (D * 8 + 16) * 4;
    static constexpr int SMEM = STAGE_BYTES > COMB_BYTES ? STAGE_BYTES : COMB_BYTES;
    static constexpr int PART = 8 * D + 16;            // floats of one chunk's state: O[8][D], m[8], l[8]
};

template <int D, int G>
__global__ void __launch_bounds__(DC_WARPS * 32) k1d_partial_kernel(Problem p, const __nv_bfloat16* __restrict__ q,
                                                                     const __nv_bfloat16* __restrict__ k,
                                                                     const __nv_bfloat16* __restrict__ v,
                                                                     float* __restrict__ part, float* __restrict__ s2out,
                                                                     int chunk, int n_chunks) {
    using C = DcCfg<D>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ci = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int64_t t = seq_pos0(p, b, KID_DECODE);  // n_q == 1: the query's position
    const int64_t j0 = (int64_t)ci * chunk;
    const int64_t j1 = min(j0 + chunk, t + 1);     // keys [j0, j1)
    const int n = j1 > j0 ? (int)(j1 - j0) : 0;
    const int n_mt = (n + 15) / 16;

    uint32_t qb[D / 16][2];
    {
        const int hh = lane >> 2;
        const bool ok = hh < G;
        const __nv_bfloat16* qrow = q + ((int64_t)(b * p.hq + g * G + (ok ? hh : 0)) * p.nq) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int d0 = ks * 16 + 2 * (lane & 3);
            qb[ks][0] = ok ? *reinterpret_cast<const uint32_t*>(qrow + d0) : 0u;
            qb[ks][1] = ok ? *reinterpret_cast<const uint32_t*>(qrow + d0 + 8) : 0u;
        }
    }
    const __nv_bfloat16* kg = k + ((int64_t)(b * p.hkv + g) * p.kv_len) * D;
    const __nv_bfloat16* vg = v + ((int64_t)(b * p.hkv + g) * p.kv_len) * D;
    float* s2g = s2out + ((int64_t)(b * p.hkv + g) * p.kv_len) * 8;
    const uint32_t s_w = smem_u32(smem) + warp * C::WARP_BYTES;
    auto load_tile = [&](int mt, int stage) {
        const uint32_t sk = s_w + stage * 2 * C::TILE, sv = sk + C::TILE;
#pragma unroll
        for (int it = 0; it < 16 * C::CH / 32; ++it) {
            const int c = it * 32 + lane;
            const int r = c / C::CH, ch = c % C::CH;
            const int64_t j = j0 + mt * 16 + r;
            const bool ok = j < j1;
            const int64_t off = (ok ? j : j0) * D + ch * 8;
            cp_async16(sk + swz<C::CH>(r, ch), kg + off, ok ? 16 : 0);
            cp_async16(sv + swz<C::CH>(r, ch), vg + off, ok ? 16 : 0);
        }
    };

    float acc[D / 16][4];
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) acc[dt][0] = acc[dt][1] = acc[dt][2] = acc[dt][3] = 0.f;
    float m_c[2] = {-INFINITY, -INFINITY}, l_c[2] = {0.f, 0.f};
    const int n_mine = n_mt > warp ? (n_mt - warp + DC_WARPS - 1) / DC_WARPS : 0;
#pragma unroll
    for (int u = 0; u < DC_NST - 1; ++u) {
        if (u < n_mine) load_tile(warp + u * DC_WARPS, u);
        cp_async_commit();
    }
    for (int u = 0; u < n_mine; ++u) {
        const int mt = warp + u * DC_WARPS;
        if (u + DC_NST - 1 < n_mine) load_tile(mt + (DC_NST - 1) * DC_WARPS, (u + DC_NST - 1) % DC_NST);
        cp_async_commit();
        cp_async_wait<DC_NST - 1>();
        __syncwarp();
        const uint32_t sk = s_w + (u % DC_NST) * 2 * C::TILE, sv = sk + C::TILE;
        float c[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a[4];
            const int mi = lane >> 3;
            ldsm_x4(a, sk + swz<C::CH>((mi & 1) * 8 + (lane & 7), 2 * ks + (mi >> 1)));
            mma16816((ks & 1) ? c2 : c, a, qb[ks]);
        }
        float s[4];
        bool row_ok[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) row_ok[r] = j0 + mt * 16 + (lane >> 2) + 8 * r < j1;
#pragma unroll
        for (int e = 0; e < 4; ++e) s[e] = row_ok[e >> 1] ? (c[e] + c2[e]) * p.scale_log2 : -INFINITY;
        // the candidates' logits for the selection: [group][j][head], heads 2*(lane%4)+{0,1}
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int64_t j = j0 + mt * 16 + (lane >> 2) + 8 * r;
            if (j <= t - p.window && j < j1)
                *reinterpret_cast<float2*>(s2g + j * 8 + 2 * (lane & 3)) = make_float2(s[2 * r], s[2 * r + 1]);
        }
        float mx[2];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            float x = fmaxf(s[cc], s[cc + 2]);
            x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
            x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
            mx[cc] = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
        }
        const bool grow = mx[0] > m_c[0] || mx[1] > m_c[1];
        if (__any_sync(0xffffffffu, grow)) {
            float alpha[2];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const float m_new = fmaxf(m_c[cc], mx[cc]);
                alpha[cc] = m_new == -INFINITY ? 1.f : ex2(m_c[cc] - m_new);
                m_c[cc] = m_new;
                l_c[cc] *= alpha[cc];
            }
#pragma unroll
            for (int dt = 0; dt < D / 16; ++dt) {
                acc[dt][0] *= alpha[0];
                acc[dt][1] *= alpha[1];
                acc[dt][2] *= alpha[0];
                acc[dt][3] *= alpha[1];
            }
        }
        float pr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float mu = m_c[e & 1] == -INFINITY ? 0.f : m_c[e & 1];
            pr[e] = ex2(s[e] - mu);
            l_c[e & 1] += pr[e];
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
    }
    cp_async_wait<0>();
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        l_c[cc] += __shfl_xor_sync(0xffffffffu, l_c[cc], 4);
        l_c[cc] += __shfl_xor_sync(0xffffffffu, l_c[cc], 8);
        l_c[cc] += __shfl_xor_sync(0xffffffffu, l_c[cc], 16);
    }
    __syncthreads();
    // merge the warps, write this chunk's state (8 head slots; heads >= G unused)
    float* comb = reinterpret_cast<float*>(smem);
    float* ot = comb + warp * (D * 8 + 16);  // [8][D] then m[8], l[8]
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int d = dt * 16 + (lane >> 2) + 8 * (e >> 1);
            const int col = 2 * (lane & 3) + (e & 1);
            ot[col * D + d] = acc[dt][e];
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
    float* pout = part + ((int64_t)(b * p.hkv + g) * n_chunks + ci) * C::PART;
    for (int u = tid; u < 8 * D; u += DC_WARPS * 32) {
        const int hh = u / D, d = u % D;
        float mm = -INFINITY;
#pragma unroll
        for (int w = 0; w < DC_WARPS; ++w) mm = fmaxf(mm, comb[w * (D * 8 + 16) + D * 8 + hh]);
        float num = 0.f;
        if (mm != -INFINITY) {
#pragma unroll
            for (int w = 0; w < DC_WARPS; ++w) {
                const float* wb = comb + w * (D * 8 + 16);
                num += ex2(wb[D * 8 + hh] - mm) * wb[hh * D + d];
            }
        }
        pout[hh * D + d] = num;
    }
    if (tid < 8) {
        float mm = -INFINITY, den = 0.f;
#pragma unroll
        for (int w = 0; w < DC_WARPS; ++w) mm = fmaxf(mm, comb[w * (D * 8 + 16) + D * 8 + tid]);
        if (mm != -INFINITY) {
#pragma unroll
            for (int w = 0; w < DC_WARPS; ++w) {
                const float* wb = comb + w * (D * 8 + 16);
                den += ex2(wb[D * 8 + tid] - mm) * wb[D * 8 + 8 + tid];
            }
        }
        pout[8 * D + tid] = mm;
        pout[8 * D + 8 + tid] = den;
    }
}

// One CTA per (sequence, KV group): exact merge of the chunk states.
template <int D, int G>
__global__ void __launch_bounds__(128) k1d_combine_kernel(Problem p, const float* __restrict__ part,
                                                          __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                                                          int n_chunks) {
    constexpr int PART = DcCfg<D>::PART;
    __shared__ float s_m[8], s_l[8];
    const int tid = threadIdx.x;
    const int g = blockIdx.x, b = blockIdx.y;
    const float* pg = part + (int64_t)(b * p.hkv + g) * n_chunks * PART;
    if (tid < G) {
        float mm = -INFINITY;
        for (int c = 0; c < n_chunks; ++c) mm = fmaxf(mm, pg[c * PART + 8 * D + tid]);
        float l = 0.f;
        for (int c = 0; c < n_chunks; ++c) {
            const float mc = pg[c * PART + 8 * D + tid];
            if (mc != -INFINITY) l += ex2(mc - mm) * pg[c * PART + 8 * D + 8 + tid];
        }
        s_m[tid] = mm;
        s_l[tid] = l;
        lse[(int64_t)(b * p.hq + g * G + tid) * p.nq] = (mm + log2f(l)) * kLn2;
    }
    __syncthreads();
    for (int u = tid; u < G * D; u += 128) {
        const int hh = u / D, d = u % D;
        const float mm = s_m[hh];
        float num = 0.f;
        for (int c = 0; c < n_chunks; ++c) {
            const float mc = pg[c * PART + 8 * D + hh];
            if (mc != -INFINITY) num += ex2(mc - mm) * pg[c * PART + hh * D + d];
        }
        out[(int64_t)(b * p.hq + g * G + hh) * p.nq * D + d] = __float2bfloat16_rn(num / s_l[hh]);
    }
}

// score_j = sum_h 2^(s2_{h,j} - lse2_h) for the candidates j <= t - window.
template <int G>
__global__ void __launch_bounds__(256) k2d_score_kernel(Problem p, const float* __restrict__ s2in,
                                                        const float* __restrict__ lse, float* __restrict__ scores,
                                                        int64_t sstride) {
    const int g = blockIdx.y, b = blockIdx.z;
    const int64_t t = seq_pos0(p, b, KID_SCORE);
    const int64_t n = t - p.window + 1;
    float l2[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) l2[hh] = lse[(int64_t)(b * p.hq + g * G + hh) * p.nq] * kLog2e;
    const float* sg = s2in + ((int64_t)(b * p.hkv + g) * p.kv_len) * 8;
    float* out = scores + (int64_t)(b * p.hkv + g) * sstride;
    for (int64_t j = (int64_t)blockIdx.x * 256 + threadIdx.x; j < n; j += (int64_t)gridDim.x * 256) {
        const float4 x0 = *reinterpret_cast<const float4*>(sg + j * 8);
        const float4 x1 = *reinterpret_cast<const float4*>(sg + j * 8 + 4);
        const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        float e[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) e[hh] = ex2(xs[hh] - l2[hh]);
#pragma unroll
        for (int w2 = 1; w2 < G; w2 *= 2)
#pragma unroll
            for (int hh = 0; hh + w2 < G; hh += 2 * w2) e[hh] += e[hh + w2];
        out[j] = e[0];
    }
}

template <int D, int G>
cudaError_t launch_decode_dg(const Problem& p, const void* q, const void* k, const void* v, void* out, float* lse,
                             float* part, float* s2, float* scores, int64_t sstride, int chunk, int n_chunks,
                             cudaStream_t st) {
    using C = DcCfg<D>;
    auto kp = k1d_partial_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kp, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    prof_begin(KID_DECODE, st);
    kp<<<dim3(n_chunks, p.hkv, p.B), DC_WARPS * 32, C::SMEM, st>>>(p, (const __nv_bfloat16*)q,
                                                                  (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                                                  part, s2, chunk, n_chunks);
    prof_end(st);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    prof_begin(KID_COMBINE, st);
    k1d_combine_kernel<D, G><<<dim3(p.hkv, p.B), 128, 0, st>>>(p, part, (__nv_bfloat16*)out, lse, n_chunks);
    prof_end(st);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (scores != nullptr) {
        const int64_t cand = p.kv_len - p.window;
        int bx = (int)((cand + 255) / 256);
        if (bx > 256) bx = 256;
        if (bx < 1) bx = 1;
        prof_begin(KID_SCORE, st);
        k2d_score_kernel<G><<<dim3(bx, p.hkv, p.B), 256, 0, st>>>(p, s2, lse, scores, sstride);
        prof_end(st);
        count_launch();
        e = cudaGetLastError();
    }
    return e;
}

template <int D>
cudaError_t launch_decode_d(const Problem& p, const void* q, const void* k, const void* v, void* out, float* lse,
                            float* part, float* s2, float* scores, int64_t sstride, int chunk, int n_chunks,
                            cudaStream_t st) {
    switch (p.hq / p.hkv) {
        case 1: return launch_decode_dg<D, 1>(p, q, k, v, out, lse, part, s2, scores, sstride, chunk, n_chunks, st);
        case 2: return launch_decode_dg<D, 2>(p, q, k, v, out, lse, part, s2, scores, sstride, chunk, n_chunks, st);
        case 4: return launch_decode_dg<D, 4>(p, q, k, v, out, lse, part, s2, scores, sstride, chunk, n_chunks, st);
        default: return launch_decode_dg<D, 8>(p, q, k, v, out, lse, part, s2, scores, sstride, chunk, n_chunks, st);
    }
}

}  // namespace

void decode_geometry(const Problem& p, int& chunk, int& n_chunks) {
    // enough CTAs to fill the machine a few times over, chunks of whole 64-key tiles
    const int64_t want = (4 * 148 + (int64_t)p.B * p.hkv - 1) / ((int64_t)p.B * p.hkv);
    int64_t c = (p.kv_len + want - 1) / want;
    c = (c + 63) / 64 * 64;
    if (c < 256) c = 256;
    chunk = (int)c;
    n_chunks = (int)((p.kv_len + c - 1) / c);
}

size_t decode_scratch_bytes(const Problem& p) {
    int chunk, n_chunks;
    decode_geometry(p, chunk, n_chunks);
    const size_t part = (size_t)p.B * p.hkv * n_chunks * (8 * p.D + 16) * 4;
    const size_t s2 = (size_t)p.B * p.hkv * p.kv_len * 8 * 4;
    return (part + 255) / 256 * 256 + (s2 + 255) / 256 * 256;
}

cudaError_t launch_decode(const Problem& p, const void* q, const void* k, const void* v, void* out, float* lse,
                          void* scratch, float* scores, int64_t sstride, cudaStream_t st) {
    int chunk, n_chunks;
    decode_geometry(p, chunk, n_chunks);
    float* part = reinterpret_cast<float*>(scratch);
    const size_t part_bytes = (size_t)p.B * p.hkv * n_chunks * (8 * p.D + 16) * 4;
    float* s2 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(scratch) + (part_bytes + 255) / 256 * 256);
    if (p.D == 64) return launch_decode_d<64>(p, q, k, v, out, lse, part, s2, scores, sstride, chunk, n_chunks, st);
    return launch_decode_d<128>(p, q, k, v, out, lse, part, s2, scores, sstride, chunk, n_chunks, st);
}

}  // namespace hs2
