// k1_full_attn.cu -- K1: causal GQA full attention with LSE (the Cross-Decoder's
// full-attention layer of HySparse2; xiawanshe.com report, section "两级KV共享":
// this layer's cache and selection are reused by the following sparse layers).
//
// One CTA = 64 query rows of one head, 4 warps x 16 rows.  K/V tiles of 64 keys
// are staged in shared memory with cp.async (double buffered, XOR-swizzled
// rows); S = Q K^T and O += P V run on the tensor cores through mma.sync
// m16n8k16 (bf16 in, fp32 accumulate); the softmax is the online (running max
// and sum) form in base 2 with the scale folded into one multiply.
#include "hs2_kernels.h"

namespace hs2 {

namespace {

template <int D>
struct K1Cfg {
    static constexpr int BM = 64;
    static constexpr int BN = 64;
    static constexpr int CH = D / 8;  // 16-byte chunks per row
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int T_BYTES = BN * D * 2;
    static constexpr int SMEM = Q_BYTES + 4 * T_BYTES;
};

template <int D>
__global__ void __launch_bounds__(128) k1_full_kernel(Problem p, const __nv_bfloat16* __restrict__ q,
                                                      const __nv_bfloat16* __restrict__ k,
                                                      const __nv_bfloat16* __restrict__ v,
                                                      __nv_bfloat16* __restrict__ out,
                                                      float* __restrict__ lse) {
    using C = K1Cfg<D>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i0 = blockIdx.x * C::BM;
    const int h = blockIdx.y, b = blockIdx.z;
    const int G = p.hq / p.hkv, g = h / G;
    const int64_t pos0 = seq_pos0(p, b, KID_FULL);
    const int i_last = min(i0 + C::BM, p.nq) - 1;
    const int64_t t_max = pos0 + i_last;
    const int n_tiles = (int)((t_max + C::BN) / C::BN);

    const __nv_bfloat16* qh = q + ((int64_t)(b * p.hq + h) * p.nq) * D;
    const __nv_bfloat16* kg = k + ((int64_t)(b * p.hkv + g) * p.kv_len) * D;
    const __nv_bfloat16* vg = v + ((int64_t)(b * p.hkv + g) * p.kv_len) * D;
    const uint32_t s_q = smem_u32(smem);
    const uint32_t s_t = s_q + C::Q_BYTES;  // stage s: K at s_t + 2s*T, V at + T

    // Q tile (rows past n_q are zero-filled)
    for (int c = tid; c < C::BM * C::CH; c += 128) {
        const int r = c / C::CH, ch = c % C::CH;
        const int i = i0 + r;
        const bool ok = i < p.nq;
        cp_async16(s_q + swz<C::CH>(r, ch), qh + (int64_t)(ok ? i : 0) * D + ch * 8, ok ? 16 : 0);
    }
    auto load_tile = [&](int kt, int stage) {
        const uint32_t sk = s_t + stage * 2 * C::T_BYTES, sv = sk + C::T_BYTES;
        for (int c = tid; c < C::BN * C::CH; c += 128) {
            const int r = c / C::CH, ch = c % C::CH;
            const int64_t j = (int64_t)kt * C::BN + r;
            const bool ok = j < p.kv_len;
            const int64_t off = (ok ? j : 0) * D + ch * 8;
            cp_async16(sk + swz<C::CH>(r, ch), kg + off, ok ? 16 : 0);
            cp_async16(sv + swz<C::CH>(r, ch), vg + off, ok ? 16 : 0);
        }
    };
    load_tile(0, 0);
    cp_async_commit();

    uint32_t qa[D / 16][4];
    float o[D / 8][4];
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
    // absolute positions of this thread's two rows (rows past n_q act as the last row)
    const int r0 = warp * 16 + (lane >> 2);
    const int64_t t_r[2] = {pos0 + min(i0 + r0, p.nq - 1), pos0 + min(i0 + r0 + 8, p.nq - 1)};

    for (int kt = 0; kt < n_tiles; ++kt) {
        if (kt + 1 < n_tiles) {
            load_tile(kt + 1, (kt + 1) & 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (kt == 0) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int mi = lane >> 3;
                ldsm_x4(qa[ks], s_q + swz<C::CH>(warp * 16 + (mi & 1) * 8 + (lane & 7), 2 * ks + (mi >> 1)));
            }
        }
        const uint32_t sk = s_t + (kt & 1) * 2 * C::T_BYTES, sv = sk + C::T_BYTES;

        // S = Q K^T for 16 rows x 64 keys
        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ks += 2) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                uint32_t bk[4];
                ldsm_x4(bk, sk + swz<C::CH>(nt * 8 + (lane & 7), 2 * ks + (lane >> 3)));
                mma16816(s[nt], qa[ks], bk);
                mma16816(s[nt], qa[ks + 1], bk + 2);
            }
        }
        // scale, causal mask, running max
        const int64_t j_base = (int64_t)kt * C::BN;
        const bool need_mask = j_base + C::BN - 1 > pos0 + i0;
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float x = s[nt][e] * p.scale_log2;
                if (need_mask) {
                    const int64_t j = j_base + nt * 8 + 2 * (lane & 3) + (e & 1);
                    if (j > t_r[e >> 1]) x = -INFINITY;
                }
                s[nt][e] = x;
                mx[e >> 1] = fmaxf(mx[e >> 1], x);
            }
        }
        float alpha[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
            const float m_new = fmaxf(m_r[r], mx[r]);
            alpha[r] = ex2(m_r[r] - m_new);
            m_r[r] = m_new;
            l_r[r] *= alpha[r];
        }
#pragma unroll
        for (int dt = 0; dt < D / 8; ++dt) {
            o[dt][0] *= alpha[0];
            o[dt][1] *= alpha[0];
            o[dt][2] *= alpha[1];
            o[dt][3] *= alpha[1];
        }
        // P = 2^(S - m), row sums, then O += P V
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float pv = ex2(s[nt][e] - m_r[e >> 1]);
                s[nt][e] = pv;
                l_r[e >> 1] += pv;
            }
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t pa[4];
            pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
            pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
            pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int dt = 0; dt < D / 8; dt += 2) {
                uint32_t bv[4];
                const int mi = lane >> 3;
                ldsm_x4_t(bv, sv + swz<C::CH>(kk * 16 + (mi & 1) * 8 + (lane & 7), dt + (mi >> 1)));
                mma16816(o[dt], pa, bv);
                mma16816(o[dt + 1], pa, bv + 2);
            }
        }
        __syncthreads();
    }

    // epilogue: normalise, write out (bf16) and lse (natural log)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
        l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
    }
    const float inv[2] = {1.f / l_r[0], 1.f / l_r[1]};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int i = i0 + r0 + 8 * r;
        if (i >= p.nq) continue;
        __nv_bfloat16* orow = out + ((int64_t)(b * p.hq + h) * p.nq + i) * D;
#pragma unroll
        for (int dt = 0; dt < D / 8; ++dt) {
            const uint32_t pk = pack_bf16(o[dt][2 * r] * inv[r], o[dt][2 * r + 1] * inv[r]);
            *reinterpret_cast<uint32_t*>(orow + dt * 8 + 2 * (lane & 3)) = pk;
        }
        if ((lane & 3) == 0) lse[(int64_t)(b * p.hq + h) * p.nq + i] = (m_r[r] + log2f(l_r[r])) * kLn2;
    }
}

template <int D>
cudaError_t launch_full_d(const Problem& p, const void* q, const void* k, const void* v, void* out,
                          float* lse, cudaStream_t st) {
    using C = K1Cfg<D>;
    auto kern = k1_full_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid((p.nq + C::BM - 1) / C::BM, p.hq, p.B);
    prof_begin(KID_FULL, st);
    kern<<<grid, 128, C::SMEM, st>>>(p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                     (const __nv_bfloat16*)v, (__nv_bfloat16*)out, lse);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_full(const Problem& p, const void* q, const void* k, const void* v, void* out,
                        float* lse, void* scratch, size_t scratch_bytes, cudaStream_t st) {
    // prefill-shaped calls run on the tcgen05 kernel; decode-shaped ones (one
    // query per sequence) on the mma.sync kernel below
    if (p.seq_len == nullptr && p.nq >= 64) return launch_full_tc(p, q, k, v, out, lse, scratch, scratch_bytes, st);
    if (p.D == 64) return launch_full_d<64>(p, q, k, v, out, lse, st);
    return launch_full_d<128>(p, q, k, v, out, lse, st);
}

}  // namespace hs2
