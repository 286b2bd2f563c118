// k0_bridge_tc.cu -- K0: KV bridging of HySparse2 (xiawanshe.com report,
// section "两级KV共享", first level "KV Bridging": the Cross-Decoder's K and V
// come from the Self-Decoder's hidden states), the projection that fills the
// shared cache the rest of the path reads.
//
//   kv (tokens x 2 H_kv D) = hidden (tokens x d_model) W_kv^T, fp32 accumulate,
//   written as bf16 straight into k_cache / v_cache [b][h][pos_b + i][d].
//
// A dense contraction, so on the 5th-generation tensor cores: one CTA = a 128
// token x 256 feature tile of the output, 6 warps:
//   warps 0-3  epilogue: thread r owns token row r (= TMEM lane r); its 256
//              fp32 accumulators are two heads' rows of K (or of V), stored as
//              two 256-byte cache rows
//   warp 4     TMA producer: 64-wide K-steps of hidden (128 x 64) and W_kv
//              (256 x 64), 4-stage ring
//   warp 5     TMEM allocator and MMA issuer (one elected lane):
//              tcgen05.mma M = 128, N = 256, K = 16, A = hidden, B = W_kv,
//              both K-major, accumulator in 256 TMEM columns
// Operand tiles are 128-byte swizzled (TMA SWIZZLE_128B).  Every wait is
// bounded; a stalled CTA reports HS2_ERR_TIMEOUT, drains and exits.
//
// Few tokens (the decode-time append: one token per sequence) leave only a few
// CTAs to stream all of W_kv.  Then the d_model range is split over blockIdx.z:
// each CTA accumulates its slice of the K-steps and writes an fp32 partial
// tile, and k0_bridge_reduce_kernel sums the partials and writes the cache rows.
#include <cudaTypedefs.h>

#include "hs2_kernels.h"
#include "tc05.cuh"

namespace hs2 {

bool make_map(CUtensorMap* m, const void* base, uint64_t x, uint64_t y, uint64_t z, uint32_t box_rows);  // k1_full_tc.cu

namespace {

constexpr int BR_BM = 128;  // token rows per CTA
constexpr int BR_BN = 256;  // output features per CTA
constexpr int BR_BK = 64;   // d_model per K-step (one 128-byte swizzle atom row)
constexpr int BR_NS = 4;    // ring stages
constexpr int BR_TMA_WARP = 4;
constexpr int BR_MMA_WARP = 5;
constexpr int BR_THREADS = 192;
constexpr int BR_ABLK = BR_BM * 128;  // one stage of hidden: 128 rows x 128 B
constexpr int BR_BBLK = BR_BN * 128;  // one stage of W_kv: 256 rows x 128 B
constexpr int BR_A_OFF = 0;
constexpr int BR_B_OFF = BR_NS * BR_ABLK;
constexpr int BR_BAR_OFF = BR_B_OFF + BR_NS * BR_BBLK;
constexpr int BR_SMEM = BR_BAR_OFF + 256 + 1024;

enum : int { BB_FULL = 0, BB_EMPTY = BR_NS, BB_DONE = 2 * BR_NS, BB_DRAIN = BB_DONE + 1, BB_COUNT = BB_DRAIN + 1 };

struct BridgeArgs {
    int64_t n_rows;       // batch * n_new
    int n_new, d_model, h_kv, head_dim;
    int64_t pos0, kv_cap;
    const int64_t* seq_pos;
    __nv_bfloat16* k_cache;
    __nv_bfloat16* v_cache;
    WsHeader* err;
    int k_per;            // K-steps per split (all of them without a split)
    float* part;          // split: fp32 partials [split][n_rows][features], else null
};

// Cache row of token m, or -1 if its sequence's rows would leave the cache
// (then the first token of the sequence reports it).
__device__ __forceinline__ int64_t bridge_row(const BridgeArgs& a, int64_t m, int64_t& b, bool report) {
    b = m / a.n_new;
    const int64_t i = m - b * a.n_new;
    const int64_t pb = a.seq_pos ? a.seq_pos[b] : a.pos0;
    if (pb < 0 || pb + a.n_new > a.kv_cap) {
        if (report) report_error(a.err, HS2_ERR_DEVICE_CHECK, KID_BRIDGE, (uint32_t)b, (uint32_t)i);
        return -1;
    }
    return pb + i;
}

__global__ void __launch_bounds__(BR_THREADS, 1) k0_bridge_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                  const __grid_constant__ CUtensorMap tm_w,
                                                                  BridgeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
    const uint32_t sA = sbase + BR_A_OFF, sB = sbase + BR_B_OFF;
    const uint32_t bars = sbase + BR_BAR_OFF;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + BR_BAR_OFF + 8 * BB_COUNT);
    tc::Abort* ab = reinterpret_cast<tc::Abort*>(sgen + BR_BAR_OFF + 8 * BB_COUNT + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t m0 = (int64_t)blockIdx.y * BR_BM;  // first token row
    const int n0 = blockIdx.x * BR_BN;               // first output feature
    const int split = blockIdx.z;
    const int kb0 = split * a.k_per;                 // first K-step of this CTA
    const int n_k = min(a.d_model / BR_BK - kb0, a.k_per);

    if (tid == 0) {
        for (int i = 0; i < BB_COUNT; ++i) tc::mbar_init(bar(i), 1);
        ab->flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == BR_MMA_WARP) tc::tmem_alloc(smem_u32(tmem_slot), BR_BN);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == BR_TMA_WARP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int kk = 0; kk < n_k; ++kk) {
                const int s = kk % BR_NS;
                if (kk >= BR_NS &&
                    !tc::mbar_wait(bar(BB_EMPTY + s), ((kk - BR_NS) / BR_NS) & 1, ab, a.err, KID_BRIDGE, 1))
                    break;
                tc::mbar_expect_tx(bar(BB_FULL + s), BR_ABLK + BR_BBLK);
                tc::tma_load_3d(sA + s * BR_ABLK, &tm_x, bar(BB_FULL + s), (kb0 + kk) * BR_BK, (int)m0, 0);
                tc::tma_load_3d(sB + s * BR_BBLK, &tm_w, bar(BB_FULL + s), (kb0 + kk) * BR_BK, n0, 0);
                issued = kk + 1;
            }
            if (ab->flag) {  // drain: every issued load lands before the CTA exits
                tc::Abort none{0};
                for (int kk = (issued > BR_NS ? issued - BR_NS : 0); kk < issued; ++kk)
                    tc::mbar_wait(bar(BB_FULL + kk % BR_NS), (kk / BR_NS) & 1, &none, nullptr, 0, 0);
            }
        }
    } else if (warp == BR_MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t ID = tc::idesc_bf16(BR_BM, BR_BN, 0, 0);  // both K-major
        const uint64_t da0 = tc::sdesc_sw128(sA, 16, 1024), db0 = tc::sdesc_sw128(sB, 16, 1024);
        bool ok = true;
        for (int kk = 0; ok && kk < n_k; ++kk) {
            const int s = kk % BR_NS;
            ok = __all_sync(~0u, tc::mbar_wait(bar(BB_FULL + s), (kk / BR_NS) & 1, ab, a.err, KID_BRIDGE, 2));
            if (!ok) break;
            tc::fence_after_sync();
            if (tc::elect_one()) {
#pragma unroll
                for (int k4 = 0; k4 < BR_BK / 16; ++k4) {
                    const uint64_t da = da0 + (uint64_t)((s * BR_ABLK + k4 * 32) >> 4);
                    const uint64_t db = db0 + (uint64_t)((s * BR_BBLK + k4 * 32) >> 4);
                    tc::mma_ss(tmem, da, db, ID, (kk > 0 || k4 > 0) ? 1u : 0u);
                }
                tc::mma_commit(bar(BB_EMPTY + s));
                if (kk == n_k - 1) tc::mma_commit(bar(BB_DONE));
            }
            __syncwarp();
        }
        if (tc::elect_one()) tc::mma_commit(bar(BB_DRAIN));
        __syncwarp();
        tc::Abort none{0};
        tc::mbar_wait(bar(BB_DRAIN), 0, &none, nullptr, 0, 0);
    } else {
        // ------------------------------------------------------------ epilogue (warps 0-3)
        const int r = tid;  // token row within the tile == TMEM lane
        const int64_t m = m0 + r;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const bool ok = __all_sync(~0u, tc::mbar_wait(bar(BB_DONE), 0, ab, a.err, KID_BRIDGE, 3));
        tc::fence_after_sync();
        // destination of this token: sequence b, cache row pos_b + i (a split
        // writes its fp32 partial row instead; the reduce places it)
        bool write = ok && m < a.n_rows;
        int64_t b = 0, row = 0;
        if (write && a.part == nullptr) {
            row = bridge_row(a, m, b, true);
            write = row >= 0;  // the whole sequence is skipped
        }
        const int hd = a.h_kv * a.head_dim;
        const bool is_v = n0 >= hd;
        __nv_bfloat16* cache = is_v ? a.v_cache : a.k_cache;
        const int f0 = is_v ? n0 - hd : n0;  // first feature within K (or V)
#pragma unroll
        for (int c = 0; c < BR_BN / 32; ++c) {
            float o[32];
            if (ok) {
                tc::tmem_ld32(tmem + lane_off + c * 32, o);
                tc::tmem_wait_ld();
            }
            if (write && a.part != nullptr) {
                float* dst = a.part + ((int64_t)split * a.n_rows + m) * (2 * a.h_kv * a.head_dim) + n0 + c * 32;
#pragma unroll
                for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
            } else if (write) {
                const int f = f0 + c * 32;  // 32 features of one head
                const int h = f / a.head_dim, d = f - h * a.head_dim;
                __nv_bfloat16* dst = cache + (((int64_t)b * a.h_kv + h) * a.kv_cap + row) * a.head_dim + d;
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 v;
                    v.x = pack_bf16(o[e], o[e + 1]);
                    v.y = pack_bf16(o[e + 2], o[e + 3]);
                    v.z = pack_bf16(o[e + 4], o[e + 5]);
                    v.w = pack_bf16(o[e + 6], o[e + 7]);
                    *reinterpret_cast<uint4*>(dst + e) = v;
                }
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == BR_MMA_WARP) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, BR_BN);
    }
}

// Sum of the n_split fp32 partials of 8 features of one token, written as bf16
// into its cache row.
__global__ void __launch_bounds__(256) k0_bridge_reduce_kernel(BridgeArgs a, int n_split) {
    const int features = 2 * a.h_kv * a.head_dim;
    const int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t m = u / (features / 8);
    if (m >= a.n_rows) return;
    const int f = (int)(u - m * (features / 8)) * 8;
    int64_t b;
    const int64_t row = bridge_row(a, m, b, f == 0);
    if (row < 0) return;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < n_split; ++s) {
        const float* src = a.part + ((int64_t)s * a.n_rows + m) * features + f;
        const float4 x = *reinterpret_cast<const float4*>(src);
        const float4 y = *reinterpret_cast<const float4*>(src + 4);
        acc[0] += x.x, acc[1] += x.y, acc[2] += x.z, acc[3] += x.w;
        acc[4] += y.x, acc[5] += y.y, acc[6] += y.z, acc[7] += y.w;
    }
    const int hd = a.h_kv * a.head_dim;
    const bool is_v = f >= hd;
    const int fl = is_v ? f - hd : f;
    const int h = fl / a.head_dim, d = fl - h * a.head_dim;
    __nv_bfloat16* cache = is_v ? a.v_cache : a.k_cache;
    uint4 v;
    v.x = pack_bf16(acc[0], acc[1]);
    v.y = pack_bf16(acc[2], acc[3]);
    v.z = pack_bf16(acc[4], acc[5]);
    v.w = pack_bf16(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(cache + ((b * a.h_kv + h) * a.kv_cap + row) * a.head_dim + d) = v;
}

}  // namespace

// Split of the K-steps for a call of n_rows tokens: enough CTAs to stream the
// weights with most SMs; 1 when the token and feature tiles already fill them.
int bridge_splits(int64_t n_rows, int d_model, int h_kv, int head_dim) {
    const int64_t ctas = (int64_t)(2 * h_kv * head_dim / BR_BN) * ((n_rows + BR_BM - 1) / BR_BM);
    const int n_k = d_model / BR_BK;
    if (ctas >= 74 || n_k < 2) return 1;
    int want = (int)(148 / ctas);
    if (want > n_k) want = n_k;
    const int per = (n_k + want - 1) / want;
    return (n_k + per - 1) / per;  // every split gets at least one K-step
}

size_t bridge_split_bytes(int64_t n_rows, int d_model, int h_kv, int head_dim) {
    const int S = bridge_splits(n_rows, d_model, h_kv, head_dim);
    return S > 1 ? (size_t)S * n_rows * 2 * h_kv * head_dim * 4 : 0;
}

cudaError_t launch_bridge(int64_t n_rows, int n_new, int d_model, int h_kv, int head_dim, int64_t pos0,
                          int64_t kv_cap, const int64_t* seq_pos, const void* hidden, const void* w_kv,
                          void* k_cache, void* v_cache, WsHeader* err, cudaStream_t st, float* part) {
    if (n_rows == 0) return cudaSuccess;
    const int features = 2 * h_kv * head_dim;
    CUtensorMap mx, mw;
    if (!make_map(&mx, hidden, (uint64_t)d_model, (uint64_t)n_rows, 1, BR_BM) ||
        !make_map(&mw, w_kv, (uint64_t)d_model, (uint64_t)features, 1, BR_BN))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k0_bridge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, BR_SMEM);
    if (e != cudaSuccess) return e;
    BridgeArgs a;
    a.n_rows = n_rows;
    a.n_new = n_new;
    a.d_model = d_model;
    a.h_kv = h_kv;
    a.head_dim = head_dim;
    a.pos0 = pos0;
    a.kv_cap = kv_cap;
    a.seq_pos = seq_pos;
    a.k_cache = reinterpret_cast<__nv_bfloat16*>(k_cache);
    a.v_cache = reinterpret_cast<__nv_bfloat16*>(v_cache);
    a.err = err;
    const int n_k = d_model / BR_BK;
    const int S = part != nullptr ? bridge_splits(n_rows, d_model, h_kv, head_dim) : 1;
    a.k_per = (n_k + S - 1) / S;
    a.part = S > 1 ? part : nullptr;
    // feature tiles fastest: CTAs of one token tile run together and share it in L2
    dim3 grid(features / BR_BN, (unsigned)((n_rows + BR_BM - 1) / BR_BM), (unsigned)S);
    prof_begin(KID_BRIDGE, st);
    k0_bridge_kernel<<<grid, BR_THREADS, BR_SMEM, st>>>(mx, mw, a);
    prof_end(st);
    count_launch();
    if (S == 1) return cudaGetLastError();
    cudaError_t e2 = cudaGetLastError();
    if (e2 != cudaSuccess) return e2;
    const int64_t threads = n_rows * (features / 8);
    prof_begin(KID_BRIDGE, st);
    k0_bridge_reduce_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(a, S);
    prof_end(st);
    count_launch();
    return cudaGetLastError();
}

}  // namespace hs2
