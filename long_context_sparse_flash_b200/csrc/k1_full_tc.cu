// k1_full_tc.cu -- K1 on the 5th-generation tensor cores: causal GQA full
// attention with LSE for the Cross-Decoder's full-attention layer of HySparse2
// (xiawanshe.com report, section "两级KV共享": this layer's cache and its token
// selection are reused by the following sparse layers).
//
// One CTA = two 128-row query tiles (A, B) of one head, 10 warps:
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread r of a
//              warpgroup owns query row r of its tile = TMEM lane r
//   warp 8     TMA producer: both Q tiles once, then K/V tiles of 64 keys
//              (3-stage ring)
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer
// Per key tile j, for each query tile X in {A, B}:
//   S_X,j (TMEM, double buffered) = Q_X K_j^T      tcgen05.mma, A = Q_X, B = K (K-major)
//   softmax X: tcgen05.ld S_X,j, scale + causal mask, running max with lazy
//   rescale (O_X is only rescaled when the max grows by more than 2^8),
//   P_X,j = 2^(S - m) as bf16 into a 128B-swizzled shared tile
//   O_X (TMEM) += P_X,j V_j                         tcgen05.mma, A = P_X, B = V (MN-major)
// The two warpgroups' softmaxes overlap with each other's MMAs, so the tensor
// core is not left idle while one tile's exponentials are computed.
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

// [z][y][x] bf16 tensor, x contiguous (= D); box 64 x box_rows x 1, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t x, uint64_t y, uint64_t z, uint32_t box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {x, y, z};
    cuuint64_t strides[2] = {x * 2, x * y * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

constexpr int PP_QT = 2;      // query tiles per CTA
constexpr int PP_BM = 128;    // rows per query tile
constexpr int PP_BN = 64;     // keys per K/V tile
constexpr int PP_NS = 3;      // K/V ring stages
constexpr int PP_TMA_WARP = 8;
constexpr int PP_MMA_WARP = 9;
constexpr int PP_THREADS = 320;
constexpr uint32_t PP_TMEM_COLS = 512;

template <int D>
struct PpCfg {
    static constexpr int KB = D / 64;                  // 64-element (128-byte) column blocks
    static constexpr int QBLK = PP_BM * 128;           // 128 rows x 128 B
    static constexpr int KBLK = PP_BN * 128;           // 64 rows x 128 B
    static constexpr int Q_OFF = 0;                    // [tile][kb] QBLK
    static constexpr int K_OFF = Q_OFF + PP_QT * KB * QBLK;
    static constexpr int V_OFF = K_OFF + PP_NS * KB * KBLK;
    static constexpr int P_OFF = V_OFF + PP_NS * KB * KBLK;   // [tile] 128 rows x 64 keys (one block)
    static constexpr int BAR_OFF = P_OFF + PP_QT * QBLK;
    static constexpr int SMEM = BAR_OFF + 256 + 1024;
    // TMEM columns: S[tile][buf] 64 each at 0..255, O[tile] D each from 256
    static constexpr int O_COL = 4 * PP_BN;
};

enum : int {
    PB_Q = 0,
    PB_KFULL = 1,
    PB_VFULL = PB_KFULL + PP_NS,
    PB_KVEMPTY = PB_VFULL + PP_NS,
    PB_SFULL = PB_KVEMPTY + PP_NS,   // [tile][buf]
    PB_SEMPTY = PB_SFULL + 4,        // [tile][buf]
    PB_PFULL = PB_SEMPTY + 4,        // [tile]
    PB_ODONE = PB_PFULL + 2,         // [tile]
    PB_DRAIN = PB_ODONE + 2,
    PB_COUNT = PB_DRAIN + 1,
};

// Row of 64 scores of one S tile from TMEM (this thread's lane); keys past
// the causal limit t are set to -inf.
__device__ __forceinline__ void load_scores(uint32_t addr, float* s, bool diag, int64_t j0, int64_t t) {
    tc::tmem_ld32(addr, s);
    tc::tmem_ld32(addr + 32, s + 32);
    tc::tmem_wait_ld();
    if (diag) {
#pragma unroll
        for (int c = 0; c < PP_BN; ++c)
            if (j0 + c > t) s[c] = -INFINITY;
    }
}

// Max of the 64 raw scores: four independent three-input max chains.
__device__ __forceinline__ float tile_max(const float* s) {
    float mc[4];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
        const float* sq = s + q4 * (PP_BN / 4);
        float a = sq[0];
#pragma unroll
        for (int c = 1; c + 1 < PP_BN / 4; c += 2) a = fmax3f(a, sq[c], sq[c + 1]);
        mc[q4] = fmaxf(a, sq[PP_BN / 4 - 1]);
    }
    return fmax3f(mc[0], mc[1], fmaxf(mc[2], mc[3]));
}

// In place s <- 2^(s * scale - m) for 64 scores, two lanes per instruction;
// returns the row sum (four packed accumulators).
__device__ __forceinline__ float exp_tile(float* s, float scale, float m) {
    const float2 sc2 = make_float2(scale, scale), nm2 = make_float2(-m, -m);
    float2 acc[4];
#pragma unroll
    for (int c = 0; c < PP_BN; c += 2) {
        float2 e = ffma2(make_float2(s[c], s[c + 1]), sc2, nm2);
        e.x = ex2(e.x);
        e.y = ex2(e.y);
        s[c] = e.x;
        s[c + 1] = e.y;
        const int a4 = (c >> 1) & 3;
        acc[a4] = (c < 8) ? e : fadd2(acc[a4], e);
    }
    const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
    return (a01.x + a01.y) + (a23.x + a23.y);
}

template <int D>
__global__ void __launch_bounds__(PP_THREADS, 1) k1_full_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                  const __grid_constant__ CUtensorMap tm_k,
                                                                  const __grid_constant__ CUtensorMap tm_v,
                                                                  Problem p, __nv_bfloat16* __restrict__ out,
                                                                  float* __restrict__ lse) {
    using C = PpCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
    const uint32_t sQ = sbase + C::Q_OFF, sK = sbase + C::K_OFF, sV = sbase + C::V_OFF, sP = sbase + C::P_OFF;
    const uint32_t bars = sbase + C::BAR_OFF;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + C::BAR_OFF + 8 * PB_COUNT);
    tc::Abort* ab = reinterpret_cast<tc::Abort*>(sgen + C::BAR_OFF + 8 * PB_COUNT + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_blk = (p.nq + PP_QT * PP_BM - 1) / (PP_QT * PP_BM);
    const int blk = n_blk - 1 - (int)blockIdx.x;  // longest causal rows first
    const int i0 = blk * PP_QT * PP_BM;
    const int h = blockIdx.y, b = blockIdx.z;
    const int G = p.hq / p.hkv, g = h / G;
    const int64_t pos0 = seq_pos0(p, b, KID_FULL);
    const int i_last = min(i0 + PP_QT * PP_BM, p.nq) - 1;
    const int n_tiles = (int)((pos0 + i_last + PP_BN) / PP_BN);

    if (tid == 0) {
        for (int i = 0; i < PB_COUNT; ++i) {
            uint32_t cnt = 1;
            if ((i >= PB_SEMPTY && i < PB_SEMPTY + 4) || (i >= PB_PFULL && i < PB_PFULL + 2)) cnt = 128;
            tc::mbar_init(bar(i), cnt);
        }
        ab->flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == PP_MMA_WARP) tc::tmem_alloc(smem_u32(tmem_slot), PP_TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == PP_TMA_WARP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const int zq = b * p.hq + h, zk = b * p.hkv + g;
            tc::mbar_expect_tx(bar(PB_Q), PP_QT * C::KB * C::QBLK);
            for (int x = 0; x < PP_QT; ++x)
                for (int kb = 0; kb < C::KB; ++kb)
                    tc::tma_load_3d(sQ + (x * C::KB + kb) * C::QBLK, &tm_q, bar(PB_Q), kb * 64, i0 + x * PP_BM, zq);
            int issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % PP_NS;
                if (j >= PP_NS &&
                    !tc::mbar_wait(bar(PB_KVEMPTY + s), ((j - PP_NS) / PP_NS) & 1, ab, p.err, KID_FULL, 1))
                    break;
                tc::mbar_expect_tx(bar(PB_KFULL + s), C::KB * C::KBLK);
                for (int kb = 0; kb < C::KB; ++kb)
                    tc::tma_load_3d(sK + (s * C::KB + kb) * C::KBLK, &tm_k, bar(PB_KFULL + s), kb * 64, j * PP_BN, zk);
                tc::mbar_expect_tx(bar(PB_VFULL + s), C::KB * C::KBLK);
                for (int kb = 0; kb < C::KB; ++kb)
                    tc::tma_load_3d(sV + (s * C::KB + kb) * C::KBLK, &tm_v, bar(PB_VFULL + s), kb * 64, j * PP_BN, zk);
                issued = j + 1;
            }
            if (ab->flag) {  // drain: every issued load lands before the CTA exits
                tc::Abort none{0};
                tc::mbar_wait(bar(PB_Q), 0, &none, nullptr, 0, 0);
                for (int j = (issued > PP_NS ? issued - PP_NS : 0); j < issued; ++j) {
                    const int s = j % PP_NS;
                    tc::mbar_wait(bar(PB_KFULL + s), (j / PP_NS) & 1, &none, nullptr, 0, 0);
                    tc::mbar_wait(bar(PB_VFULL + s), (j / PP_NS) & 1, &none, nullptr, 0, 0);
                }
            }
        }
    } else if (warp == PP_MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop and its waits (votes keep it converged);
        // one elected lane issues the MMAs and their commits.
        constexpr uint32_t ID_S = tc::idesc_bf16(PP_BM, PP_BN, 0, 0);  // A = Q, B = K: both K-major
        constexpr uint32_t ID_O = tc::idesc_bf16(PP_BM, D, 0, 1);      // A = P K-major, B = V MN-major
        // descriptors of the first block of each operand; a byte offset o moves
        // the start address field by o / 16
        const uint64_t dq0 = tc::sdesc_sw128(sQ, 16, 1024), dk0 = tc::sdesc_sw128(sK, 16, 1024);
        const uint64_t dp0 = tc::sdesc_sw128(sP, 16, 1024), dv0 = tc::sdesc_sw128(sV, C::KBLK, 1024);
        bool ok = __all_sync(~0u, tc::mbar_wait(bar(PB_Q), 0, ab, p.err, KID_FULL, 2));
        for (int j = 0; ok && j <= n_tiles; ++j) {
            if (j < n_tiles) {
                const int s = j % PP_NS, sb = j & 1;
                ok = __all_sync(~0u, tc::mbar_wait(bar(PB_KFULL + s), (j / PP_NS) & 1, ab, p.err, KID_FULL, 3));
                for (int x = 0; ok && x < PP_QT; ++x) {
                    if (j >= 2)
                        ok = __all_sync(~0u, tc::mbar_wait(bar(PB_SEMPTY + 2 * x + sb), ((j - 2) >> 1) & 1, ab, p.err,
                                                           KID_FULL, 4));
                    if (!ok) break;
                    tc::fence_after_sync();
                    if (tc::elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t da = dq0 + (uint64_t)(((x * C::KB + (kk >> 2)) * C::QBLK + (kk & 3) * 32) >> 4);
                            const uint64_t db = dk0 + (uint64_t)(((s * C::KB + (kk >> 2)) * C::KBLK + (kk & 3) * 32) >> 4);
                            tc::mma_ss(tmem + (2 * x + sb) * PP_BN, da, db, ID_S, kk > 0);
                        }
                        tc::mma_commit(bar(PB_SFULL + 2 * x + sb));
                    }
                    __syncwarp();
                }
                if (!ok) break;
            }
            if (j >= 1) {
                const int jp = j - 1, sp = jp % PP_NS;
                ok = __all_sync(~0u, tc::mbar_wait(bar(PB_VFULL + sp), (jp / PP_NS) & 1, ab, p.err, KID_FULL, 5));
                for (int x = 0; ok && x < PP_QT; ++x) {
                    ok = __all_sync(~0u, tc::mbar_wait(bar(PB_PFULL + x), jp & 1, ab, p.err, KID_FULL, 6));
                    if (!ok) break;
                    tc::fence_after_sync();
                    if (tc::elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < PP_BN / 16; ++kk) {
                            const uint64_t da = dp0 + (uint64_t)((x * C::QBLK + kk * 32) >> 4);
                            const uint64_t db = dv0 + (uint64_t)((sp * C::KB * C::KBLK + kk * 2048) >> 4);
                            tc::mma_ss(tmem + C::O_COL + x * D, da, db, ID_O, (jp > 0 || kk > 0) ? 1u : 0u);
                        }
                        tc::mma_commit(bar(PB_ODONE + x));
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (tc::elect_one()) tc::mma_commit(bar(PB_KVEMPTY + sp));
                __syncwarp();
            }
        }
        // every issued MMA completes before TMEM is released
        if (tc::elect_one()) tc::mma_commit(bar(PB_DRAIN));
        __syncwarp();
        tc::Abort none{0};
        tc::mbar_wait(bar(PB_DRAIN), 0, &none, nullptr, 0, 0);
    } else {
        // ------------------------------------------------------------ softmax (warps 0-7)
        const int x = warp >> 2;                // query tile of this warpgroup
        const int r = tid & 127;                // row within the tile == TMEM lane
        const int64_t t = pos0 + min(i0 + x * PP_BM + r, p.nq - 1);
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_col = 2 * x * PP_BN, o_col = C::O_COL + x * D;
        const uint32_t sPx = sP + x * C::QBLK;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        float s[PP_BN];
        for (int j = 0; j < n_tiles && ok; ++j) {
            const int sb = j & 1;
            ok = tc::mbar_wait(bar(PB_SFULL + 2 * x + sb), (j >> 1) & 1, ab, p.err, KID_FULL, 7);
            if (!ok) break;
            tc::fence_after_sync();
            const uint32_t s_addr = tmem + lane_off + s_col + sb * PP_BN;
            const int64_t j0 = (int64_t)j * PP_BN;
            const bool diag = j0 + PP_BN - 1 > t;
            load_scores(s_addr, s, diag, j0, t);
            tc::fence_before_sync();
            tc::mbar_arrive(bar(PB_SEMPTY + 2 * x + sb));
            const float mt = tile_max(s) * p.scale_log2;
            bool waited_o = false;
            if (mt > m + 8.f) {
                // the running max grew by more than 2^8: rescale l and O
                const float alpha = ex2(m - mt);
                if (j > 0) {
                    ok = tc::mbar_wait(bar(PB_ODONE + x), (j - 1) & 1, ab, p.err, KID_FULL, 8);
                    if (!ok) break;
                    waited_o = true;
                    tc::fence_after_sync();
                    float o[32];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        tc::tmem_ld32(tmem + lane_off + o_col + c * 32, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= alpha;
                        tc::tmem_st32(tmem + lane_off + o_col + c * 32, o);
                    }
                    tc::tmem_wait_st();
                }
                l *= alpha;
                m = mt;
            }
            l += exp_tile(s, p.scale_log2, m);
            // the P tile is free once the previous P V product has completed
            if (j > 0 && !waited_o) {
                ok = tc::mbar_wait(bar(PB_ODONE + x), (j - 1) & 1, ab, p.err, KID_FULL, 9);
                if (!ok) break;
            }
            // P row r: 64 keys = one 128-byte row of the swizzled block
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const float* v8 = s + ch * 8;
                uint4 v;
                v.x = pack_bf16(v8[0], v8[1]);
                v.y = pack_bf16(v8[2], v8[3]);
                v.z = pack_bf16(v8[4], v8[5]);
                v.w = pack_bf16(v8[6], v8[7]);
                const uint32_t addr = sPx + r * 128 + ((ch ^ (r & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                             "r"(v.w)
                             : "memory");
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(PB_PFULL + x));
        }
        // epilogue: O / l -> out (bf16), lse
        if (ok) ok = tc::mbar_wait(bar(PB_ODONE + x), (n_tiles - 1) & 1, ab, p.err, KID_FULL, 10);
        if (ok) {
            tc::fence_after_sync();
            const int i = i0 + x * PP_BM + r;
            const float inv = 1.f / l;
            __nv_bfloat16* orow = out + ((int64_t)(b * p.hq + h) * p.nq + i) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                tc::tmem_ld32(tmem + lane_off + o_col + c * 32, o);
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
    if (warp == PP_MMA_WARP) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, PP_TMEM_COLS);
    }
}

template <int D>
cudaError_t launch_full_tc_d(const Problem& p, const void* q, const void* k, const void* v, void* out, float* lse,
                             cudaStream_t st) {
    using C = PpCfg<D>;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, D, (uint64_t)p.nq, (uint64_t)p.B * p.hq, PP_BM) ||
        !make_map(&mk, k, D, (uint64_t)p.kv_len, (uint64_t)p.B * p.hkv, PP_BN) ||
        !make_map(&mv, v, D, (uint64_t)p.kv_len, (uint64_t)p.B * p.hkv, PP_BN))
        return cudaErrorInvalidValue;
    auto kern = k1_full_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid((p.nq + PP_QT * PP_BM - 1) / (PP_QT * PP_BM), p.hq, p.B);
    prof_begin(KID_FULL, st);
    kern<<<grid, PP_THREADS, C::SMEM, st>>>(mq, mk, mv, p, (__nv_bfloat16*)out, lse);
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
