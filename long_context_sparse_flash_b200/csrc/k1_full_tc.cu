// k1_full_tc.cu -- K1 on the 5th-generation tensor cores: causal GQA full
// attention with LSE for the Cross-Decoder's full-attention layer of HySparse2
// (xiawanshe.com report, section "两级KV共享": this layer's cache and its token
// selection are reused by the following sparse layers).
//
// One CTA = two 128-row query tiles (A, B) of one head, 12 warps (384 threads):
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread r of a
//              warpgroup owns query row r of its tile = TMEM lane r
//   warp 8     TMA producer: both Q tiles once, then K and V tiles of 128 keys
//              (separate rings, since K of a tile is consumed a step before V)
//   warp 9     TMEM allocator and MMA issuer (one elected lane)
//   warps 10-11 idle; with warps 8-9 they form the warpgroup that hands its
//              registers to the softmax warpgroups (setmaxnreg)
// Per key tile j, for each query tile X in {A, B}:
//   S_X,j (TMEM, 128 columns) = Q_X K_j^T           tcgen05.mma, A = Q_X, B = K (smem, K-major)
//   softmax X: tcgen05.ld S_X,j, causal mask, running max with lazy rescale
//   (O_X is only rescaled when the max grows by more than 2^8),
//   P_X,j = 2^(S - m) as bf16 pairs, tcgen05.st over the first half of S_X
//   O_X (TMEM) += P_X,j V_j                          tcgen05.mma, A = P_X (TMEM), B = V (smem, MN-major)
// Keeping P in tensor memory leaves the shared-memory operand reads of the
// P V product to V alone; the two tiles' softmaxes alternate with each other's
// MMAs, so the tensor core is not left idle while one tile's exponentials run.
// Operand tiles are 128-byte swizzled (TMA SWIZZLE_128B), rows of 64 bf16.
// Every wait is bounded (tc::mbar_wait): a stalled CTA reports HS2_ERR_TIMEOUT
// through the error word, drains its own copies, frees its TMEM and exits.
//
// The K/V buffer may hold one slice of a longer context (context parallelism:
// positions shifted by the slice's first key).  A query past the buffer's last
// key sees all of it; a query before its first key sees none (output 0, LSE
// -inf).  Long causal rows with few CTAs split their key range over blockIdx.z
// and merge the parts exactly (k1_split_combine_kernel).
#include <cudaTypedefs.h>

#include "exp2_poly.cuh"
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
constexpr int PP_BN = 128;    // keys per K/V tile
constexpr int PP_TMA_WARP = 8;
constexpr int PP_MMA_WARP = 9;
constexpr int PP_THREADS = 384;   // warps 10-11 only complete the third warpgroup
// register budgets after the split: softmax warpgroups up, the rest down
constexpr uint32_t PP_REG_SOFTMAX = 208, PP_REG_OTHER = 80;
constexpr uint32_t PP_TMEM_COLS = 512;

template <int D>
struct PpCfg {
    static constexpr int KB = D / 64;                  // 64-element (128-byte) column blocks
    static constexpr int BLK = 128 * 128;              // one block: 128 rows x 128 B
    // ring stages of K and V tiles: K(j+1) and V(j) may only load once the MMAs
    // of tile j-NS have freed their slots, and a 64 KB tile pair from L2 takes
    // about one tile period to land; at D = 128 shared memory holds one more
    // 32 KB stage, which goes to K (2-3% faster at a 1M context)
    static constexpr int NSK = D == 64 ? 4 : 3, NSV = D == 64 ? 4 : 2;
    static constexpr int Q_OFF = 0;                    // [tile][kb] BLK
    static constexpr int K_OFF = Q_OFF + PP_QT * KB * BLK;
    static constexpr int V_OFF = K_OFF + NSK * KB * BLK;
    static constexpr int BAR_OFF = V_OFF + NSV * KB * BLK;
    static constexpr int SMEM = BAR_OFF + 256 + 1024;
    // TMEM columns: S[tile] 128 each at 0 and 128 (P[tile], 128 bf16 keys =
    // 64 columns, overwrites the first half of S[tile] once it has been read),
    // O[tile] D each from 256
    static constexpr int O_COL = PP_QT * PP_BN;
};

enum : int {
    PB_Q = 0,
    PB_KFULL = 1,
    PB_VFULL = PB_KFULL + 4,
    PB_KEMPTY = PB_VFULL + 4,
    PB_VEMPTY = PB_KEMPTY + 4,
    PB_SFULL = PB_VEMPTY + 4,   // [tile]
    PB_PFULL = PB_SFULL + 2,    // [tile], 128 arrivals
    PB_ODONE = PB_PFULL + 2,    // [tile]
    PB_DRAIN = PB_ODONE + 2,
    PB_COUNT = PB_DRAIN + 1,
};

// This thread's row of one 128-key S tile from TMEM; keys past the causal
// limit t are set to -inf.
__device__ __forceinline__ void load_scores(uint32_t addr, float* s, bool diag, int64_t j0, int64_t t) {
#pragma unroll
    for (int c = 0; c < PP_BN / 32; ++c) tc::tmem_ld32(addr + 32 * c, s + 32 * c);
    tc::tmem_wait_ld();
    if (diag) {
#pragma unroll
        for (int c = 0; c < PP_BN; ++c)
            if (j0 + c > t) s[c] = -INFINITY;
    }
}

// Max of the raw scores: four independent three-input max chains.
__device__ __forceinline__ float tile_max(const float* s) {
    constexpr int L = PP_BN / 4;
    float mc[4];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
        const float* sq = s + q4 * L;
        float a = sq[0];
#pragma unroll
        for (int c = 1; c + 1 < L; c += 2) a = fmax3f(a, sq[c], sq[c + 1]);
        mc[q4] = fmaxf(a, sq[L - 1]);
    }
    return fmax3f(mc[0], mc[1], fmaxf(mc[2], mc[3]));
}

// p = 2^(s * scale - m) for the row's 128 scores, two lanes per instruction,
// packed to bf16 pairs in place (s[0..63] hold the pairs afterwards); returns the
// row sum of the fp32 values (four packed accumulators).  One pair in PP_POLY_EVERY
// is computed on the FMA pipe (degree-5 polynomial, the accuracy of the hardware
// ex2): the special-function unit's ex2 rate otherwise equals the tensor core's
// rate for this kernel, so the unit would cap it.
constexpr int PP_POLY_EVERY = 8;
__device__ __forceinline__ float exp_pack_tile(float* s, float scale, float m) {
    const float2 sc2 = make_float2(scale, scale), nm2 = make_float2(-m, -m);
    float2 acc[4];
#pragma unroll
    for (int c = 0; c < PP_BN; c += 2) {
        float2 e = ffma2(make_float2(s[c], s[c + 1]), sc2, nm2);
        if ((c >> 1) % PP_POLY_EVERY == PP_POLY_EVERY - 1) {
            e = exp2_poly5_x2(e);
        } else {
            e.x = ex2(e.x);
            e.y = ex2(e.y);
        }
        const int a4 = (c >> 1) & 3;
        acc[a4] = (c < 8) ? e : fadd2(acc[a4], e);
        s[c >> 1] = __uint_as_float(pack_bf16(e.x, e.y));
    }
    const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
    return (a01.x + a01.y) + (a23.x + a23.y);
}

template <int D>
__global__ void __launch_bounds__(PP_THREADS, 1) k1_full_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                  const __grid_constant__ CUtensorMap tm_k,
                                                                  const __grid_constant__ CUtensorMap tm_v,
                                                                  Problem p, __nv_bfloat16* __restrict__ out,
                                                                  float* __restrict__ lse, int n_split,
                                                                  float* __restrict__ part_o,
                                                                  float* __restrict__ part_l) {
    using C = PpCfg<D>;
    constexpr int NSK = C::NSK, NSV = C::NSV;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
    const uint32_t sQ = sbase + C::Q_OFF, sK = sbase + C::K_OFF, sV = sbase + C::V_OFF;
    const uint32_t bars = sbase + C::BAR_OFF;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + C::BAR_OFF + 8 * PB_COUNT);
    tc::Abort* ab = reinterpret_cast<tc::Abort*>(sgen + C::BAR_OFF + 8 * PB_COUNT + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_blk = (p.nq + PP_QT * PP_BM - 1) / (PP_QT * PP_BM);
    const int blk = n_blk - 1 - (int)blockIdx.x;  // longest causal rows first
    const int i0 = blk * PP_QT * PP_BM;
    const int h = blockIdx.y, b = (int)blockIdx.z / n_split, split = (int)blockIdx.z % n_split;
    const int G = p.hq / p.hkv, g = h / G;
    const int64_t pos0 = seq_pos0(p, b, KID_FULL);
    const int i_last = min(i0 + PP_QT * PP_BM, p.nq) - 1;
    // key tiles of the causal range; with a split, this CTA takes the split-th of
    // n_split contiguous parts, tiles jt0 .. jt0 + n_tiles - 1 (loop indices below
    // are local, tile jt0 + j is read)
    // (a query may sit before the buffer's first key or past its last one when the
    // buffer holds one slice of a longer context: its keys are those of the slice)
    const int64_t t_last = min(pos0 + i_last, p.kv_len - 1);
    const int n_all = t_last < 0 ? 0 : (int)((t_last + PP_BN) / PP_BN);
    const int per = (n_all + n_split - 1) / n_split;
    const int jt0 = min(split * per, n_all);
    const int n_tiles = min(per, n_all - jt0);

    if (tid == 0) {
        for (int i = 0; i < PB_COUNT; ++i) tc::mbar_init(bar(i), (i == PB_PFULL || i == PB_PFULL + 1) ? 128u : 1u);
        ab->flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == PP_MMA_WARP) tc::tmem_alloc(smem_u32(tmem_slot), PP_TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 8) {
      tc::setmaxnreg_dec<PP_REG_OTHER>();
      if (warp == PP_TMA_WARP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const int zq = b * p.hq + h, zk = b * p.hkv + g;
            tc::mbar_expect_tx(bar(PB_Q), PP_QT * C::KB * C::BLK);
            for (int x = 0; x < PP_QT; ++x)
                for (int kb = 0; kb < C::KB; ++kb)
                    tc::tma_load_3d(sQ + (x * C::KB + kb) * C::BLK, &tm_q, bar(PB_Q), kb * 64, i0 + x * PP_BM, zq);
            // K of tile j is needed one step before V of tile j: issue K(j), then V(j - 1)
            int k_issued = 0, v_issued = 0;
            bool ok = true;
            for (int j = 0; ok && j <= n_tiles; ++j) {
                if (j < n_tiles) {
                    const int s = j % NSK;
                    if (j >= NSK) ok = tc::mbar_wait(bar(PB_KEMPTY + s), ((j - NSK) / NSK) & 1, ab, p.err, KID_FULL, 1);
                    if (!ok) break;
                    tc::mbar_expect_tx(bar(PB_KFULL + s), C::KB * C::BLK);
                    for (int kb = 0; kb < C::KB; ++kb)
                        tc::tma_load_3d(sK + (s * C::KB + kb) * C::BLK, &tm_k, bar(PB_KFULL + s), kb * 64,
                                        (jt0 + j) * PP_BN, zk);
                    k_issued = j + 1;
                }
                if (j >= 1) {
                    const int jv = j - 1, s = jv % NSV;
                    if (jv >= NSV) ok = tc::mbar_wait(bar(PB_VEMPTY + s), ((jv - NSV) / NSV) & 1, ab, p.err, KID_FULL, 2);
                    if (!ok) break;
                    tc::mbar_expect_tx(bar(PB_VFULL + s), C::KB * C::BLK);
                    for (int kb = 0; kb < C::KB; ++kb)
                        tc::tma_load_3d(sV + (s * C::KB + kb) * C::BLK, &tm_v, bar(PB_VFULL + s), kb * 64,
                                        (jt0 + jv) * PP_BN, zk);
                    v_issued = jv + 1;
                }
            }
            if (!ok || ab->flag) {  // drain: every issued load lands before the CTA exits
                tc::Abort none{0};
                tc::mbar_wait(bar(PB_Q), 0, &none, nullptr, 0, 0);
                for (int j = (k_issued > NSK ? k_issued - NSK : 0); j < k_issued; ++j)
                    tc::mbar_wait(bar(PB_KFULL + j % NSK), (j / NSK) & 1, &none, nullptr, 0, 0);
                for (int j = (v_issued > NSV ? v_issued - NSV : 0); j < v_issued; ++j)
                    tc::mbar_wait(bar(PB_VFULL + j % NSV), (j / NSV) & 1, &none, nullptr, 0, 0);
            }
        }
      } else if (warp == PP_MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop and its waits (votes keep it converged);
        // one elected lane issues the MMAs and their commits.  Per key tile j:
        //   O_A += P_A,j V_j ; S_A,j+1 = Q_A K_j+1 ; O_B += P_B,j V_j ; S_B,j+1 = Q_B K_j+1
        // so the tensor core runs one tile's products while the other tile's
        // softmax runs.  S_X,j+1 overwrites the columns P_X,j is read from; the
        // MMAs of this thread execute in issue order, so P V reads P first.
        constexpr uint32_t ID_S = tc::idesc_bf16(PP_BM, PP_BN, 0, 0);  // A = Q, B = K: both K-major
        constexpr uint32_t ID_O = tc::idesc_bf16(PP_BM, D, 0, 1);      // A = P (TMEM), B = V MN-major
        // descriptors of the first block of each operand; a byte offset o moves
        // the start address field by o / 16
        const uint64_t dq0 = tc::sdesc_sw128(sQ, 16, 1024), dk0 = tc::sdesc_sw128(sK, 16, 1024);
        const uint64_t dv0 = tc::sdesc_sw128(sV, C::BLK, 1024);
        auto issue_s = [&](int x, int j) {
            const int s = j % NSK;
            if (tc::elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t da = dq0 + (uint64_t)(((x * C::KB + (kk >> 2)) * C::BLK + (kk & 3) * 32) >> 4);
                    const uint64_t db = dk0 + (uint64_t)(((s * C::KB + (kk >> 2)) * C::BLK + (kk & 3) * 32) >> 4);
                    tc::mma_ss(tmem + x * PP_BN, da, db, ID_S, kk > 0);
                }
                tc::mma_commit(bar(PB_SFULL + x));
            }
            __syncwarp();
        };
        auto issue_pv = [&](int x, int j) {
            const int s = j % NSV;
            if (tc::elect_one()) {
#pragma unroll
                for (int kk = 0; kk < PP_BN / 16; ++kk) {
                    const uint64_t db = dv0 + (uint64_t)((s * C::KB * C::BLK + kk * 2048) >> 4);
                    tc::mma_ts(tmem + C::O_COL + x * D, tmem + x * PP_BN + kk * 8, db, ID_O, (j > 0 || kk > 0) ? 1u : 0u);
                }
            }
            __syncwarp();
        };
        auto commit = [&](int i) {
            if (tc::elect_one()) tc::mma_commit(bar(i));
            __syncwarp();
        };
        bool ok = __all_sync(~0u, tc::mbar_wait(bar(PB_Q), 0, ab, p.err, KID_FULL, 3));
        if (ok && n_tiles > 0) ok = __all_sync(~0u, tc::mbar_wait(bar(PB_KFULL), 0, ab, p.err, KID_FULL, 4));
        if (ok && n_tiles > 0) {
            tc::fence_after_sync();
            issue_s(0, 0);
            issue_s(1, 0);
            commit(PB_KEMPTY);
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
            const int s = j % NSV, s1 = (j + 1) % NSK;
            const bool more = j + 1 < n_tiles;
            ok = __all_sync(~0u, tc::mbar_wait(bar(PB_VFULL + s), (j / NSV) & 1, ab, p.err, KID_FULL, 5));
            if (ok && more)
                ok = __all_sync(~0u, tc::mbar_wait(bar(PB_KFULL + s1), ((j + 1) / NSK) & 1, ab, p.err, KID_FULL, 6));
            for (int x = 0; ok && x < PP_QT; ++x) {
                ok = __all_sync(~0u, tc::mbar_wait(bar(PB_PFULL + x), j & 1, ab, p.err, KID_FULL, 7));
                if (!ok) break;
                tc::fence_after_sync();
                issue_pv(x, j);
                if (more)
                    issue_s(x, j + 1);
                else
                    commit(PB_ODONE + x);
            }
            if (!ok) break;
            commit(PB_VEMPTY + s);
            if (more) commit(PB_KEMPTY + s1);
        }
        // every issued MMA completes before TMEM is released
        commit(PB_DRAIN);
        tc::Abort none{0};
        tc::mbar_wait(bar(PB_DRAIN), 0, &none, nullptr, 0, 0);
      }
    } else {
        tc::setmaxnreg_inc<PP_REG_SOFTMAX>();
        // ------------------------------------------------------------ softmax (warps 0-7)
        const int x = warp >> 2;                // query tile of this warpgroup
        const int r = tid & 127;                // row within the tile == TMEM lane
        const int64_t t = min(pos0 + min(i0 + x * PP_BM + r, p.nq - 1), p.kv_len - 1);  // last key of the row
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + x * PP_BN, o_addr = tmem + lane_off + C::O_COL + x * D;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        float s[PP_BN];
        for (int j = 0; j < n_tiles && ok; ++j) {
            // (votes keep each warp's tcgen05 loads converged on an aborted wait)
            ok = __all_sync(~0u, tc::mbar_wait(bar(PB_SFULL + x), j & 1, ab, p.err, KID_FULL, 8));
            if (!ok) break;
            tc::fence_after_sync();
            const int64_t j0 = (int64_t)(jt0 + j) * PP_BN;
            load_scores(s_addr, s, j0 + PP_BN - 1 > t, j0, t);
            const float mt = tile_max(s) * p.scale_log2;
            const bool grow = mt > m + 8.f;
            if (__any_sync(0xffffffffu, grow)) {
                // the running max of a row grew by more than 2^8: rescale its l
                // and O.  tcgen05.ld / st are warp-collective, so the whole warp
                // runs the O pass and the rows that keep their max scale by 1.
                // The commit behind S_X,j covers O_X += P_X,j-1 V_j-1: O is final.
                const float alpha = grow ? ex2(m - mt) : 1.f;
                if (j > 0) {
                    float o[32];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        tc::tmem_ld32(o_addr + c * 32, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= alpha;
                        tc::tmem_st32(o_addr + c * 32, o);
                    }
                }
                if (grow) {
                    l *= alpha;
                    m = mt;
                }
            }
            // (m stays -inf only while every key so far is masked, which a split
            // can start with: those exponentials are 0)
            l += exp_pack_tile(s, p.scale_log2, m == -INFINITY ? 0.f : m);
            // P_X,j (bf16 pairs) over the first 64 columns of S_X
            tc::tmem_st32(s_addr, s);
            tc::tmem_st32(s_addr + 32, s + 32);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(PB_PFULL + x));
        }
        // epilogue: O / l -> out (bf16), lse; with a split, the part's O / l (fp32)
        // and base-2 log-sum-exp for the merge
        if (ok && n_tiles > 0) ok = __all_sync(~0u, tc::mbar_wait(bar(PB_ODONE + x), 0, ab, p.err, KID_FULL, 9));
        if (ok && n_split > 1) {
            tc::fence_after_sync();
            const int i = i0 + x * PP_BM + r;
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const int64_t prow = (((int64_t)split * p.B + b) * p.hq + h) * p.nq + i;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                if (n_tiles > 0) {
                    tc::tmem_ld32(o_addr + c * 32, o);
                    tc::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0.f;
                }
                if (i < p.nq) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(part_o + prow * D + c * 32 + e) =
                            make_float4(o[e] * inv, o[e + 1] * inv, o[e + 2] * inv, o[e + 3] * inv);
                }
            }
            if (i < p.nq) part_l[prow] = l > 0.f ? m + log2f(l) : -INFINITY;
        } else if (ok) {
            tc::fence_after_sync();
            const int i = i0 + x * PP_BM + r;
            const float inv = l > 0.f ? 1.f / l : 0.f;  // l = 0: the row has no key in the buffer
            __nv_bfloat16* orow = out + ((int64_t)(b * p.hq + h) * p.nq + i) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                if (n_tiles > 0) {
                    tc::tmem_ld32(o_addr + c * 32, o);
                    tc::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0.f;
                }
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
            if (i < p.nq) lse[(int64_t)(b * p.hq + h) * p.nq + i] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == PP_MMA_WARP) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, PP_TMEM_COLS);
    }
}

// Exact merge of the split parts of each row: with part lse2_s = m_s + log2(l_s)
// and part output O_s = (sum p v) / l_s, out = sum_s 2^(lse2_s - M) O_s / L and
// lse = ln 2 (M + log2 L), M = max_s lse2_s, L = sum_s 2^(lse2_s - M).
// One warp per (sequence, head, query) row.
template <int D>
__global__ void __launch_bounds__(256) k1_split_combine_kernel(Problem p, int n_split, const float* __restrict__ part_o,
                                                               const float* __restrict__ part_l,
                                                               __nv_bfloat16* __restrict__ out,
                                                               float* __restrict__ lse) {
    const int64_t rows = (int64_t)p.B * p.hq * p.nq;
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, part_l[(int64_t)s * rows + row]);
    constexpr int E = D / 32;  // elements per lane
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    float L = 0.f;
    for (int s = 0; s < n_split; ++s) {
        const float ls = part_l[(int64_t)s * rows + row];
        const float w = ls == -INFINITY ? 0.f : ex2(ls - M);
        L += w;
        const float* o = part_o + ((int64_t)s * rows + row) * D + lane * E;
        if constexpr (E == 4) {
            const float4 v = *reinterpret_cast<const float4*>(o);
            acc[0] += w * v.x, acc[1] += w * v.y, acc[2] += w * v.z, acc[3] += w * v.w;
        } else {
            const float2 v = *reinterpret_cast<const float2*>(o);
            acc[0] += w * v.x, acc[1] += w * v.y;
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16* orow = out + row * D + lane * E;
    if constexpr (E == 4) {
        uint2 v;
        v.x = pack_bf16(acc[0] * inv, acc[1] * inv);
        v.y = pack_bf16(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2*>(orow) = v;
    } else {
        *reinterpret_cast<uint32_t*>(orow) = pack_bf16(acc[0] * inv, acc[1] * inv);
    }
    if (lane == 0) lse[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

template <int D>
cudaError_t launch_full_tc_d(const Problem& p, const void* q, const void* k, const void* v, void* out, float* lse,
                             int n_split, float* part_o, float* part_l, cudaStream_t st) {
    using C = PpCfg<D>;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, D, (uint64_t)p.nq, (uint64_t)p.B * p.hq, PP_BM) ||
        !make_map(&mk, k, D, (uint64_t)p.kv_len, (uint64_t)p.B * p.hkv, PP_BN) ||
        !make_map(&mv, v, D, (uint64_t)p.kv_len, (uint64_t)p.B * p.hkv, PP_BN))
        return cudaErrorInvalidValue;
    auto kern = k1_full_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    // the register split must fit in what the CTA is launched with, or the
    // increase would wait for registers that never come
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if ((long)fa.numRegs * PP_THREADS < 256L * PP_REG_SOFTMAX + 128L * PP_REG_OTHER) return cudaErrorInvalidConfiguration;
    dim3 grid((p.nq + PP_QT * PP_BM - 1) / (PP_QT * PP_BM), p.hq, p.B * n_split);
    prof_begin(KID_FULL, st);
    kern<<<grid, PP_THREADS, C::SMEM, st>>>(mq, mk, mv, p, (__nv_bfloat16*)out, lse, n_split, part_o, part_l);
    if (n_split > 1) {
        const int64_t rows = (int64_t)p.B * p.hq * p.nq;
        k1_split_combine_kernel<D><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(
            p, n_split, part_o, part_l, (__nv_bfloat16*)out, lse);
        count_launch();
    }
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

// Parts the key range of each full-attention CTA is split into.  Calls with
// few, very long CTAs (a short chunk appended to a long cache) leave part of
// the last wave of 148 SMs idle; splitting each CTA's keys into S parts (each
// at least 256 tiles) and merging the parts exactly fills the waves.  S is the
// smallest value whose idle fraction of the last wave is at least 2 points
// better than S = 1 (deterministic: the workspace size depends on it).
int full_tc_splits(const Problem& p) {
    if (p.seq_len != nullptr || p.nq < 64) return 1;
    const int64_t ctas = (int64_t)((p.nq + PP_QT * PP_BM - 1) / (PP_QT * PP_BM)) * p.hq * p.B;
    // key tiles of the shortest query block (keys past the buffer's end do not exist)
    const int64_t first_keys = min(p.q_pos0 + (p.nq < PP_QT * PP_BM ? p.nq : PP_QT * PP_BM), p.kv_len);
    const int64_t min_tiles = first_keys > 0 ? (first_keys + PP_BN - 1) / PP_BN : 0;
    auto idle = [](int64_t n) {
        const int64_t waves = (n + 147) / 148;
        return (double)(waves * 148 - n) / (double)(waves * 148);
    };
    int best = 1;
    double best_idle = idle(ctas);
    for (int S = 2; S <= 4; ++S) {
        if (min_tiles / S < 256) break;
        const double f = idle(ctas * S);
        if (f < best_idle - 0.02) {
            best = S;
            best_idle = f;
        }
    }
    return best;
}

size_t full_tc_split_scratch_bytes(const Problem& p) {
    const int S = full_tc_splits(p);
    if (S <= 1) return 0;
    const size_t rows = (size_t)p.B * p.hq * p.nq;
    return (size_t)S * rows * ((size_t)p.D * 4 + 4) + 256;
}

cudaError_t launch_full_tc(const Problem& p, const void* q, const void* k, const void* v, void* out, float* lse,
                           void* scratch, size_t scratch_bytes, cudaStream_t st) {
    int S = full_tc_splits(p);
    float *part_o = nullptr, *part_l = nullptr;
    if (S > 1 && scratch != nullptr && scratch_bytes >= full_tc_split_scratch_bytes(p)) {
        const size_t rows = (size_t)p.B * p.hq * p.nq;
        part_o = reinterpret_cast<float*>(scratch);
        part_l = part_o + (size_t)S * rows * p.D;
    } else {
        S = 1;
    }
    if (p.D == 64) return launch_full_tc_d<64>(p, q, k, v, out, lse, S, part_o, part_l, st);
    return launch_full_tc_d<128>(p, q, k, v, out, lse, S, part_o, part_l, st);
}

}  // namespace hs2
