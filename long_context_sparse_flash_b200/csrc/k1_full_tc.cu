// k1_full_tc.cu -- K1 on the 5th-generation tensor cores: causal GQA full
// attention with LSE for the Cross-Decoder's full-attention layer of HySparse2
// (xiawanshe.com report, section "两级KV共享": this layer's cache and its token
// selection are reused by the following sparse layers).
//
// One CTA = 128 query rows of one head, 6 warps:
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r
//   warp 4     TMA producer: Q once, then K/V tiles of 128 keys (2 stages)
//   warp 5     TMEM allocator and single-thread tcgen05.mma issuer
// Per key tile j:
//   S_j (TMEM, double buffered) = Q K_j^T        tcgen05.mma, A = Q, B = K (K-major)
//   softmax: tcgen05.ld S_j, scale + causal mask, running max with lazy
//   rescale (O is only rescaled when the max grows by more than 2^8),
//   P_j = 2^(S - m) as bf16 into a 128B-swizzled shared tile
//   O (TMEM) += P_j V_j                          tcgen05.mma, A = P, B = V (MN-major)
// Operand tiles are 128-byte swizzled (TMA SWIZZLE_128B), rows of 64 bf16.
// Every wait is bounded (tc::mbar_wait): a stalled CTA reports HS2_ERR_TIMEOUT
// through the error word, drains its own copies, frees its TMEM and exits.
#include <cudaTypedefs.h>

#include "hs2_kernels.h"
#include "tc05.cuh"

namespace hs2 {

// ---------------------------------------------------------------------------
// host

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// [z][y][x] bf16 tensor, x contiguous (= D); box 64 x 128 x 1, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t x, uint64_t y, uint64_t z) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {x, y, z};
    cuuint64_t strides[2] = {x * 2, x * y * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

constexpr int TC_BM = 128;   // query rows per CTA
constexpr int TC_BN = 128;   // keys per tile
constexpr int TC_NS = 2;     // K/V pipeline stages
constexpr int TC_THREADS = 192;
constexpr uint32_t TC_TMEM_COLS = 512;

template <int D>
struct TcCfg {
    static constexpr int KB = D / 64;                 // 64-element (128-byte) column blocks
    static constexpr int BLK = 128 * 128;             // bytes of one 128-row x 128-byte block
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + KB * BLK;
    static constexpr int V_OFF = K_OFF + TC_NS * KB * BLK;
    static constexpr int P_OFF = V_OFF + TC_NS * KB * BLK;
    static constexpr int BAR_OFF = P_OFF + 2 * BLK;   // P: 128 keys = 2 blocks
    static constexpr int SMEM = BAR_OFF + 256 + 1024; // barriers + alignment slack
    static constexpr int O_COL = 2 * TC_BN;           // TMEM: S0 [0,128), S1 [128,256), O [256, 256+D)
};

// barrier slots (8 bytes each) in the barrier area
enum : int {
    B_Q = 0,
    B_KFULL = 1,               // + stage
    B_VFULL = B_KFULL + TC_NS,  // + stage
    B_KVEMPTY = B_VFULL + TC_NS,
    B_SFULL = B_KVEMPTY + TC_NS,  // + buffer (2)
    B_SEMPTY = B_SFULL + 2,
    B_PFULL = B_SEMPTY + 2,
    B_ODONE = B_PFULL + 1,
    B_DRAIN = B_ODONE + 1,     // the MMA thread's final commit
    B_COUNT = B_DRAIN + 1,
};

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 1) k1_full_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                  const __grid_constant__ CUtensorMap tm_k,
                                                                  const __grid_constant__ CUtensorMap tm_v,
                                                                  Problem p, __nv_bfloat16* __restrict__ out,
                                                                  float* __restrict__ lse) {
    using C = TcCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
    const uint32_t sQ = sbase + C::Q_OFF, sK = sbase + C::K_OFF, sV = sbase + C::V_OFF, sP = sbase + C::P_OFF;
    const uint32_t bars = sbase + C::BAR_OFF;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + C::BAR_OFF + 8 * B_COUNT);
    tc::Abort* ab = reinterpret_cast<tc::Abort*>(sgen + C::BAR_OFF + 8 * B_COUNT + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_qt = (p.nq + TC_BM - 1) / TC_BM;
    const int qt = n_qt - 1 - (int)blockIdx.x;  // longest causal rows first
    const int i0 = qt * TC_BM;
    const int h = blockIdx.y, b = blockIdx.z;
    const int G = p.hq / p.hkv, g = h / G;
    const int64_t pos0 = seq_pos0(p, b, KID_FULL);
    const int i_last = min(i0 + TC_BM, p.nq) - 1;
    const int n_tiles = (int)((pos0 + i_last + TC_BN) / TC_BN);

    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            uint32_t cnt = 1;
            if (i == B_SEMPTY || i == B_SEMPTY + 1 || i == B_PFULL) cnt = 128;
            tc::mbar_init(bar(i), cnt);
        }
        ab->flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 5) tc::tmem_alloc(smem_u32(tmem_slot), TC_TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const int zq = b * p.hq + h, zk = b * p.hkv + g;
            tc::mbar_expect_tx(bar(B_Q), C::KB * C::BLK);
            for (int kb = 0; kb < C::KB; ++kb) tc::tma_load_3d(sQ + kb * C::BLK, &tm_q, bar(B_Q), kb * 64, i0, zq);
            int issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % TC_NS;
                if (j >= TC_NS &&
                    !tc::mbar_wait(bar(B_KVEMPTY + s), ((j - TC_NS) / TC_NS) & 1, ab, p.err, KID_FULL, 1))
                    break;
                tc::mbar_expect_tx(bar(B_KFULL + s), C::KB * C::BLK);
                for (int kb = 0; kb < C::KB; ++kb)
                    tc::tma_load_3d(sK + (s * C::KB + kb) * C::BLK, &tm_k, bar(B_KFULL + s), kb * 64, j * TC_BN, zk);
                tc::mbar_expect_tx(bar(B_VFULL + s), C::KB * C::BLK);
                for (int kb = 0; kb < C::KB; ++kb)
                    tc::tma_load_3d(sV + (s * C::KB + kb) * C::BLK, &tm_v, bar(B_VFULL + s), kb * 64, j * TC_BN, zk);
                issued = j + 1;
            }
            // drain: every issued load has landed before the CTA can exit
            if (ab->flag) {
                tc::Abort none{0};
                tc::mbar_wait(bar(B_Q), 0, &none, nullptr, 0, 0);
                for (int j = (issued > TC_NS ? issued - TC_NS : 0); j < issued; ++j) {
                    const int s = j % TC_NS;
                    tc::mbar_wait(bar(B_KFULL + s), (j / TC_NS) & 1, &none, nullptr, 0, 0);
                    tc::mbar_wait(bar(B_VFULL + s), (j / TC_NS) & 1, &none, nullptr, 0, 0);
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_S = tc::idesc_bf16(128, TC_BN, 0, 0);  // A = Q, B = K: both K-major
            constexpr uint32_t ID_O = tc::idesc_bf16(128, D, 0, 1);      // A = P K-major, B = V MN-major
            bool ok = tc::mbar_wait(bar(B_Q), 0, ab, p.err, KID_FULL, 2);
            for (int j = 0; ok && j <= n_tiles; ++j) {
                if (j < n_tiles) {
                    const int s = j % TC_NS, sb = j & 1;
                    ok = tc::mbar_wait(bar(B_KFULL + s), (j / TC_NS) & 1, ab, p.err, KID_FULL, 3);
                    if (ok && j >= 2) ok = tc::mbar_wait(bar(B_SEMPTY + sb), ((j - 2) >> 1) & 1, ab, p.err, KID_FULL, 4);
                    if (!ok) break;
                    tc::fence_after_sync();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
                        const uint64_t da = tc::sdesc_sw128(sQ + off, 16, 1024);
                        const uint64_t db = tc::sdesc_sw128(sK + s * C::KB * C::BLK + off, 16, 1024);
                        tc::mma_ss(tmem + sb * TC_BN, da, db, ID_S, kk > 0);
                    }
                    tc::mma_commit(bar(B_SFULL + sb));
                }
                if (j >= 1) {
                    const int jp = j - 1, sp = jp % TC_NS;
                    ok = tc::mbar_wait(bar(B_PFULL), jp & 1, ab, p.err, KID_FULL, 5);
                    if (ok) ok = tc::mbar_wait(bar(B_VFULL + sp), (jp / TC_NS) & 1, ab, p.err, KID_FULL, 6);
                    if (!ok) break;
                    tc::fence_after_sync();
#pragma unroll
                    for (int kk = 0; kk < TC_BN / 16; ++kk) {
                        const uint64_t da = tc::sdesc_sw128(sP + (kk >> 2) * C::BLK + (kk & 3) * 32, 16, 1024);
                        const uint64_t db = tc::sdesc_sw128(sV + sp * C::KB * C::BLK + kk * 2048, C::BLK, 1024);
                        tc::mma_ss(tmem + C::O_COL, da, db, ID_O, (jp > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(bar(B_ODONE));
                    tc::mma_commit(bar(B_KVEMPTY + sp));
                }
            }
            // every issued MMA completes before TMEM is released
            tc::mma_commit(bar(B_DRAIN));
            tc::Abort none{0};
            tc::mbar_wait(bar(B_DRAIN), 0, &none, nullptr, 0, 0);
        }
    } else {
        // ------------------------------------------------------------ softmax (warps 0-3)
        const int r = tid;  // query row within the tile == TMEM lane
        const int64_t t = pos0 + min(i0 + r, p.nq - 1);
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        float s[TC_BN];
        for (int j = 0; j < n_tiles && ok; ++j) {
            const int sb = j & 1;
            ok = tc::mbar_wait(bar(B_SFULL + sb), (j >> 1) & 1, ab, p.err, KID_FULL, 7);
            if (!ok) break;
            tc::fence_after_sync();
#pragma unroll
            for (int c = 0; c < TC_BN / 32; ++c) tc::tmem_ld32(tmem + lane_off + sb * TC_BN + c * 32, s + c * 32);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(B_SEMPTY + sb));
            // scale, causal mask, tile max
            const int64_t j0 = (int64_t)j * TC_BN;
            float mt = -INFINITY;
            if (j0 + TC_BN - 1 > t) {
#pragma unroll
                for (int c = 0; c < TC_BN; ++c) {
                    s[c] = (j0 + c <= t) ? s[c] * p.scale_log2 : -INFINITY;
                    mt = fmaxf(mt, s[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < TC_BN; ++c) {
                    s[c] *= p.scale_log2;
                    mt = fmaxf(mt, s[c]);
                }
            }
            bool waited_o = false;
            if (mt > m + 8.f) {
                // the running max grew by more than 2^8: rescale l and O
                const float alpha = ex2(m - mt);
                if (j > 0) {
                    ok = tc::mbar_wait(bar(B_ODONE), (j - 1) & 1, ab, p.err, KID_FULL, 8);
                    if (!ok) break;
                    waited_o = true;
                    tc::fence_after_sync();
                    float o[32];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        tc::tmem_ld32(tmem + lane_off + C::O_COL + c * 32, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= alpha;
                        tc::tmem_st32(tmem + lane_off + C::O_COL + c * 32, o);
                    }
                    tc::tmem_wait_st();
                }
                l *= alpha;
                m = mt;
            }
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < TC_BN; ++c) {
                s[c] = ex2(s[c] - m);
                rs += s[c];
            }
            l += rs;
            // P buffer is free once the previous P V product has completed
            if (j > 0 && !waited_o) {
                ok = tc::mbar_wait(bar(B_ODONE), (j - 1) & 1, ab, p.err, KID_FULL, 9);
                if (!ok) break;
            }
            // P row r -> two 128-row x 128-byte blocks (keys 0-63, 64-127), swizzled
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const float* x = s + kb * 64 + ch * 8;
                    uint4 v;
                    v.x = pack_bf16(x[0], x[1]);
                    v.y = pack_bf16(x[2], x[3]);
                    v.z = pack_bf16(x[4], x[5]);
                    v.w = pack_bf16(x[6], x[7]);
                    const uint32_t addr = sP + kb * C::BLK + r * 128 + ((ch ^ (r & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                                 "r"(v.w)
                                 : "memory");
                }
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(B_PFULL));
        }
        // epilogue: O / l -> out (bf16), lse
        if (ok) ok = tc::mbar_wait(bar(B_ODONE), (n_tiles - 1) & 1, ab, p.err, KID_FULL, 10);
        if (ok) {
            tc::fence_after_sync();
            const int i = i0 + r;
            const float inv = 1.f / l;
            __nv_bfloat16* orow = out + ((int64_t)(b * p.hq + h) * p.nq + i) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                tc::tmem_ld32(tmem + lane_off + C::O_COL + c * 32, o);
                tc::tmem_wait_ld();
                if (i < p.nq) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 v;
                        v.x = pack_bf16(o[e] * inv, o[e + 1] * inv);
                        v.y = pack_bf16(o[e + 2] * inv, o[e + 3] * inv);
                        v.z = pack_bf16(o[e + 4] * inv, o[e + 5] * inv);
                        v.w = pack_bf16(o[e + 6] * inv, o[e + 7] * inv);
                        *reinterpret_cast<uint4*>(orow + c * 32 + e) = v;
                    }
                }
            }
            if (i < p.nq) lse[(int64_t)(b * p.hq + h) * p.nq + i] = (m + log2f(l)) * kLn2;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, TC_TMEM_COLS);
    }
}

template <int D>
cudaError_t launch_full_tc_d(const Problem& p, const void* q, const void* k, const void* v, void* out, float* lse,
                             cudaStream_t st) {
    using C = TcCfg<D>;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, D, (uint64_t)p.nq, (uint64_t)p.B * p.hq) ||
        !make_map(&mk, k, D, (uint64_t)p.kv_len, (uint64_t)p.B * p.hkv) ||
        !make_map(&mv, v, D, (uint64_t)p.kv_len, (uint64_t)p.B * p.hkv))
        return cudaErrorInvalidValue;
    auto kern = k1_full_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid((p.nq + TC_BM - 1) / TC_BM, p.hq, p.B);
    prof_begin(KID_FULL, st);
    kern<<<grid, TC_THREADS, C::SMEM, st>>>(mq, mk, mv, p, (__nv_bfloat16*)out, lse);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_full_tc(const Problem& p, const void* q, const void* k, const void* v, void* out, float* lse,
                           cudaStream_t st) {
    if (p.D == 64) return launch_full_tc_d<64>(p, q, k, v, out, lse, st);
    return launch_full_tc_d<128>(p, q, k, v, out, lse, st);
}

}  // namespace hs2
