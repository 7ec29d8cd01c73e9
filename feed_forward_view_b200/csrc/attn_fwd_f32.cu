// attn_fwd_f32.cu -- the fp32 mode of the attention: softmax(Q K^T / 8) V with
// fp32 q_hat, k, v in and fp32 out, to about fp32 accuracy, on the bf16
// tensor cores.
//
// ("Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V", Section V slides of the
//  VGGT paper-report deck. The fp32 mode answers the vggt-jax README's
//  precision study: its attention runs in FP32 -- TF32x3 Triton kernels -- for
//  parity with the FP32 reference.)
//
// Every fp32 operand x is carried as two bf16 terms, x_hi = bf16(x) and
// x_lo = bf16(x - x_hi), which represent x to about 2^-17 relative. A product
// a b is then a_hi b_hi + a_hi b_lo + a_lo b_hi (the dropped a_lo b_lo is about
// 2^-18 a b), each term a bf16 MMA with fp32 accumulation:
//   S    = Q_hi K_hi^T + Q_hi K_lo^T + Q_lo K_hi^T          (3 x 4 K-steps, N = 96)
//   [O|l] += P_hi [V_hi|1] + P_lo [V_hi|1] + P_hi [V_lo]    (3 x 6 K-steps, N = 80/80/64)
// The row sum l comes from the ones column of the first two products (l =
// sum of P_hi + P_lo, the P that multiplies V). The exponentials must be good
// to ~2^-22: 6 of every 8 score pairs go to MUFU ex2 (that accuracy), 2 to a
// degree-5 minimax polynomial on the FMA pipe (worst relative error 2.3e-7,
// fit_exp2_poly.py), so the two units share the work (measured: +3% over
// MUFU only at 36 909 tokens; 3/8 and 4/8 are no better).
//
// One CTA per 128-row query tile of one head. Warps: 0 TMA producer (K_hi,
// K_lo, V_hi, V_lo of 96 keys into a 4-slot ring), 1 MMA issuer, 2-3 idle,
// 4-11 softmax (2 per TMEM lane quarter, 48 score columns each). Tensor
// memory: Q_hi [0, 32), Q_lo [32, 64), S [64, 160), P_hi [160, 208),
// P_lo [208, 256), [O | l] [256, 336). The softmax warps and the issuer meet
// once per key block exactly as in the bf16 kernel (attn_fwd.cu): right after
// loading S_j the softmax warps arrive on bar_c (P_{j-1} written, S free; the
// first warp has checked that K_{j+1} landed), and on that signal the issuer
// issues PV_{j-1} and S_{j+1}. No row maximum either: the prologue bounds
// every score to [-8, 8] (see attn_fwd.cu).
//
// Every wait is bounded; on timeout the CTA records it in the device status
// word, stops issuing, drains what it has in flight and frees its tensor
// memory.
#include <cuda_bf16.h>

#include "attn_common.cuh"

namespace vggt {
namespace {

using attn::drain_wait;
using attn::make_map;
using attn::Waiter;

constexpr int kBM = 128;                          // query rows per CTA
constexpr int kBN = 96;                           // keys per block
constexpr int kStages = 4;                        // K/V ring depth
constexpr int kTileBytes = kBN * kHeadDim * 2;    // one 96 x 64 bf16 tile, 12 KB
constexpr int kOCols = kHeadDim + 16;             // O (64) and the row-sum block
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 128 + 32 * kSoftmaxWarps;  // 384
constexpr int kCols = 48;                           // score columns per softmax thread
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQHi = 0, kColQLo = 32, kColS = 64, kColPHi = 160, kColPLo = 208, kColO = 256;
static_assert(kColO + kOCols <= kTmemCols, "tensor memory columns");

constexpr float kScaleLog2 = 0.125f * 1.4426950408889634f;  // log2(e) / sqrt(64)

// 2^f ~ sum c_i f^i on [-1/2, 1/2], degree 5 (Remez, fit_exp2_poly.py);
// evaluated after the Cody-Waite split x = j + f (j = round(x) by adding
// 1.5 * 2^23), 2^j applied to the exponent field.
constexpr float kE5C0 = 1.000000119e+00f;
constexpr float kE5C1 = 6.931469440e-01f;
constexpr float kE5C2 = 2.402212024e-01f;
constexpr float kE5C3 = 5.550713092e-02f;
constexpr float kE5C4 = 9.675540961e-03f;
constexpr float kE5C5 = 1.327647245e-03f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kFmaPer8 = 2;                 // of every 8 score pairs, on the FMA pipe

// 2^a, 2^b on the FMA pipe (|a|, |b| <= 125), packed f32x2 arithmetic.
__device__ __forceinline__ void exp2_pair_fma(float a, float b, float& pa, float& pb) {
    const uint64_t magic2 = f2_pack(kRoundMagic, kRoundMagic);
    const uint64_t x = f2_pack(a, b);
    const uint64_t t = f2_add(x, magic2);                          // j in the low mantissa bits
    const uint64_t nj = f2_fma(t, f2_pack(-1.0f, -1.0f), magic2);  // -j, exact
    const uint64_t f = f2_add(x, nj);                              // x - j, exact, |f| <= 1/2
    uint64_t y = f2_fma(f2_pack(kE5C5, kE5C5), f, f2_pack(kE5C4, kE5C4));
    y = f2_fma(y, f, f2_pack(kE5C3, kE5C3));
    y = f2_fma(y, f, f2_pack(kE5C2, kE5C2));
    y = f2_fma(y, f, f2_pack(kE5C1, kE5C1));
    y = f2_fma(y, f, f2_pack(kE5C0, kE5C0));
    uint32_t q0, q1, t0, t1;
    u2_unpack(y, q0, q1);
    u2_unpack(t, t0, t1);
    pa = __uint_as_float(q0 + (t0 << 23));
    pb = __uint_as_float(q1 + (t1 << 23));
}

struct SharedStorage {
    uint8_t kv[kStages][4][kTileBytes];  // [slot][K_hi, K_lo, V_hi, V_lo], 128B-swizzled
    uint8_t ones[kTileBytes];            // [1, 0, ..., 0] per key row, 128B-swizzled
    uint64_t bar_kvfull[kStages];
    uint64_t bar_kvempty[kStages];
    uint64_t bar_q;      // Q_hi / Q_lo in tensor memory
    uint64_t bar_s;      // S_j computed
    uint64_t bar_c;      // P_{j-1} written and S_j read
    uint64_t bar_pfree;  // PV_j finished
    uint64_t bar_o;      // every MMA finished (once)
    uint32_t tmem_base;
    int abort;
};
constexpr size_t kSmemBytes = sizeof(SharedStorage) + 1024;  // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory beyond the per-CTA limit");

struct Params {
    const float* q_hat;  // fp32, head planes q_stride rows apart
    float* out;          // [n_seg*q_len, H, 64]
    int* status;
    long long wait_limit;
    long long q_stride;
    int q_len, k_len, H;
    int tiles_per_seg;
};

// hi/lo bf16 terms of two fp32 values, packed low half first.
__device__ __forceinline__ void split_pair(float a, float b, uint32_t& hi, uint32_t& lo) {
    const float ah = __bfloat162float(__float2bfloat16_rn(a));
    const float bh = __bfloat162float(__float2bfloat16_rn(b));
    hi = pack_bf16x2(ah, bh);
    lo = pack_bf16x2(a - ah, b - bh);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_f32_kernel(const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo,
                    const __grid_constant__ CUtensorMap tm_vhi, const __grid_constant__ CUtensorMap tm_vlo,
                    const Params prm) {
    extern __shared__ uint8_t smem_raw[];
    SharedStorage& sm = *reinterpret_cast<SharedStorage*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int warp = __shfl_sync(0xFFFFFFFFu, static_cast<int>(threadIdx.x >> 5), 0);
    const int lane = threadIdx.x & 31;
    const int seg = blockIdx.x / prm.tiles_per_seg;
    const int tile = blockIdx.x - seg * prm.tiles_per_seg;
    const int h = blockIdx.y;
    const int k_row0 = seg * prm.k_len;
    const int nkb = (prm.k_len + kBN - 1) / kBN;
    const int last_valid = prm.k_len - (nkb - 1) * kBN;

    const uint32_t bar_kvfull0 = smem_u32(&sm.bar_kvfull[0]);
    const uint32_t bar_kvempty0 = smem_u32(&sm.bar_kvempty[0]);
    const uint32_t bar_q = smem_u32(&sm.bar_q);
    const uint32_t bar_s = smem_u32(&sm.bar_s);
    const uint32_t bar_c = smem_u32(&sm.bar_c);
    const uint32_t bar_pfree = smem_u32(&sm.bar_pfree);
    const uint32_t bar_o = smem_u32(&sm.bar_o);
    const uint32_t kv_smem0 = smem_u32(sm.kv[0][0]);
    const uint32_t ones_smem = smem_u32(sm.ones);
    auto bar_kvfull = [&](int s) { return bar_kvfull0 + 8u * s; };
    auto bar_kvempty = [&](int s) { return bar_kvempty0 + 8u * s; };
    // tile i (0 K_hi, 1 K_lo, 2 V_hi, 3 V_lo) of slot s
    auto tile_smem = [&](int s, int i) { return kv_smem0 + static_cast<uint32_t>(kTileBytes) * (4 * s + i); };

    attn::fill_ones_tile(sm.ones, kTileBytes, kThreads);
    fence_proxy_async_smem();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_kvfull(s), 1);
            mbar_init(bar_kvempty(s), 1);
        }
        mbar_init(bar_q, kSoftmaxWarps);
        mbar_init(bar_s, 1);
        mbar_init(bar_c, kSoftmaxWarps);
        mbar_init(bar_pfree, 1);
        mbar_init(bar_o, 1);
        sm.abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_khi);
        tma_prefetch_desc(&tm_klo);
        tma_prefetch_desc(&tm_vhi);
        tma_prefetch_desc(&tm_vlo);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = __shfl_sync(0xFFFFFFFFu, sm.tmem_base, 0);
    const Waiter wait{prm.wait_limit, &sm.abort, prm.status};

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int n_issued = 0;
            for (int j = 0; j < nkb; ++j) {
                const int s = j % kStages;
                const uint32_t use = j / kStages;
                if (use > 0 && !wait(bar_kvempty(s), (use - 1) & 1)) break;
                mbar_arrive_expect_tx(bar_kvfull(s), 4 * kTileBytes);
                const int row = k_row0 + j * kBN;
                tma_load_3d(tile_smem(s, 0), &tm_khi, bar_kvfull(s), 0, row, h);
                tma_load_3d(tile_smem(s, 1), &tm_klo, bar_kvfull(s), 0, row, h);
                tma_load_3d(tile_smem(s, 2), &tm_vhi, bar_kvfull(s), 0, h, row);
                tma_load_3d(tile_smem(s, 3), &tm_vlo, bar_kvfull(s), 0, h, row);
                ++n_issued;
            }
            for (int j = max(0, n_issued - kStages); j < n_issued; ++j)
                drain_wait(bar_kvfull(j % kStages), (j / kStages) & 1, prm.wait_limit);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, false);
        constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, kOCols, true);
        constexpr uint32_t idesc_o64 = idesc_bf16_f32(kBM, kHeadDim, true);
        auto uwait = [&](uint32_t bar, uint32_t parity) {
            return __all_sync(0xFFFFFFFFu, wait(bar, parity)) != 0;
        };
        const uint32_t s_tm = tmem + kColS, o_tm = tmem + kColO;
        const uint32_t qh_tm = tmem + kColQHi, ql_tm = tmem + kColQLo;
        const uint32_t ph_tm = tmem + kColPHi, pl_tm = tmem + kColPLo;
        // S_j: 3 products x 4 steps of 16 head dims (8 TMEM columns of Q, 32
        // bytes of each 128-byte K row)
        auto issue_s = [&](int j) {
            const int s = j % kStages;
            const uint64_t kh = smem_desc_sw128(tile_smem(s, 0), 16, 1024);
            const uint64_t kl = smem_desc_sw128(tile_smem(s, 1), 16, 1024);
            if (elect_one()) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(s_tm, qh_tm + 8 * kk, kh + static_cast<uint64_t>((kk * 32) >> 4), idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(s_tm, qh_tm + 8 * kk, kl + static_cast<uint64_t>((kk * 32) >> 4), idesc_s, 1u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(s_tm, ql_tm + 8 * kk, kh + static_cast<uint64_t>((kk * 32) >> 4), idesc_s, 1u);
                mma_commit(bar_s);
            }
            __syncwarp();
        };
        // PV_j: 3 products x 6 steps of 16 keys; the first two carry the ones
        // column (the B operand's second 64-column block, a leading byte
        // offset away from the V_hi tile)
        auto issue_pv = [&](int j) {
            const int s = j % kStages;
            const uint32_t vh_addr = tile_smem(s, 2);
            const uint64_t vh = smem_desc_sw128(vh_addr, ones_smem - vh_addr, 1024);
            const uint64_t vl = smem_desc_sw128(tile_smem(s, 3), 16, 1024);
            if (elect_one()) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 6; ++kk)
                    mma_ts(o_tm, ph_tm + 8 * kk, vh + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_o,
                           (j > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 6; ++kk)
                    mma_ts(o_tm, pl_tm + 8 * kk, vh + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_o, 1u);
#pragma unroll
                for (int kk = 0; kk < 6; ++kk)
                    mma_ts(o_tm, ph_tm + 8 * kk, vl + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_o64, 1u);
                mma_commit(bar_pfree);
                mma_commit(bar_kvempty(s));
            }
            __syncwarp();
        };
        bool ok = uwait(bar_q, 0) && uwait(bar_kvfull(0), 0);
        if (ok) issue_s(0);
        ok = ok && uwait(bar_c, 0);  // S_0 read (and K_1 landed)
        if (ok && nkb > 1) issue_s(1);
        for (int j = 0; ok && j < nkb; ++j) {
            if (!uwait(bar_c, (j + 1) & 1)) break;  // P_j written, S_{j+1} read, K_{j+2} landed
            issue_pv(j);
            if (j + 2 < nkb) issue_s(j + 2);
        }
        if (elect_one()) mma_commit(bar_o);
        __syncwarp();
        drain_wait(bar_o, 0, prm.wait_limit);
    } else if (warp >= 4) {
        // ------------------------------------------------------ softmax
        const int half = (warp - 4) >> 2;  // score columns [48*half, +48)
        const int quarter = warp & 3;      // TMEM lanes [32*quarter, +32)
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        auto uwait = [&](uint32_t bar, uint32_t parity) {
            return __all_sync(0xFFFFFFFFu, wait(bar, parity)) != 0;
        };
        const int row_in_seg = tile * kBM + row;
        const bool row_live = row_in_seg < prm.q_len;
        const long long grow = static_cast<long long>(seg) * prm.q_len + row_in_seg;
        // Q into tensor memory: this thread's 32 dims of its row, scaled by
        // log2(e)/8 in fp32, as hi and lo bf16 terms (16 columns each).
        {
            uint32_t qh[16], ql[16];
            if (row_live) {
                const float4* src = reinterpret_cast<const float4*>(
                    prm.q_hat + (static_cast<long long>(h) * prm.q_stride + grow) * kHeadDim + 32 * half);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 w = __ldg(src + i);
                    split_pair(w.x * kScaleLog2, w.y * kScaleLog2, qh[2 * i], ql[2 * i]);
                    split_pair(w.z * kScaleLog2, w.w * kScaleLog2, qh[2 * i + 1], ql[2 * i + 1]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) qh[i] = ql[i] = 0u;
            }
            tmem_st16(lane_base + kColQHi + 16 * half, qh);
            tmem_st16(lane_base + kColQLo + 16 * half, ql);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_q);
        }
        bool ok = true;
        for (int j = 0; j < nkb; ++j) {
            if (!uwait(bar_s, j & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[kCols];
            {
                uint32_t r[kCols];
                tmem_ld48(lane_base + kColS + kCols * half, r);
#pragma unroll
                for (int i = 0; i < kCols; ++i) s[i] = __uint_as_float(r[i]);
            }
            if (quarter == 0 && half == 0 && j + 1 < nkb &&
                !uwait(bar_kvfull((j + 1) % kStages), ((j + 1) / kStages) & 1)) {
                ok = false;
                break;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_c);
            if (j == nkb - 1 && last_valid < kBN) {
                const int valid = last_valid - kCols * half;
#pragma unroll
                for (int c = 0; c < kCols; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            uint32_t ph[kCols / 2], pl[kCols / 2];
            if (j == nkb - 1) {  // masked columns are -inf: MUFU only (2^-inf = 0)
#pragma unroll
                for (int c = 0; c < kCols / 2; ++c)
                    split_pair(ex2_approx(s[2 * c]), ex2_approx(s[2 * c + 1]), ph[c], pl[c]);
            } else {
#pragma unroll
                for (int c = 0; c < kCols / 2; ++c) {
                    float pa, pb;
                    if (c % 8 < kFmaPer8) {
                        exp2_pair_fma(s[2 * c], s[2 * c + 1], pa, pb);
                    } else {
                        pa = ex2_approx(s[2 * c]);
                        pb = ex2_approx(s[2 * c + 1]);
                    }
                    split_pair(pa, pb, ph[c], pl[c]);
                }
            }
            if (j > 0 && !uwait(bar_pfree, (j - 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            tmem_st24(lane_base + kColPHi + (kCols / 2) * half, ph);
            tmem_st24(lane_base + kColPLo + (kCols / 2) * half, pl);
        }
        if (ok) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_c);
        }
        if (ok && uwait(bar_o, 0)) {
            tc_fence_after();
            uint32_t o[33];  // this thread's 32 output dims and l (column 64)
            tmem_ld32_1(lane_base + kColO + 32 * half, lane_base + kColO + kHeadDim, o);
            const float l = __uint_as_float(o[32]);
            if (row_live) {
                if (!(l > 0.0f && l <= 3.0e38f)) atomicOr(prm.status, kStatusRange);
                float4* dst = reinterpret_cast<float4*>(prm.out + (grow * prm.H + h) * kHeadDim + 32 * half);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(__fdiv_rn(__uint_as_float(o[4 * i]), l), __fdiv_rn(__uint_as_float(o[4 * i + 1]), l),
                                         __fdiv_rn(__uint_as_float(o[4 * i + 2]), l), __fdiv_rn(__uint_as_float(o[4 * i + 3]), l));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- host

}  // namespace

cudaError_t launch_attention_f32(const AttnProblemF32& p, int* status, long long wait_limit, cudaStream_t stream) {
    if (p.n_seg <= 0 || p.H <= 0 || p.q_len <= 0 || p.k_len <= 0) return cudaSuccess;
    const uint64_t nk = static_cast<uint64_t>(p.n_seg) * p.k_len;
    const uint64_t row_bytes = kHeadDim * 2;
    const uint64_t ks = static_cast<uint64_t>(p.k_stride);
    CUtensorMap tm_khi, tm_klo, tm_vhi, tm_vlo;
    if (!make_map(&tm_khi, p.k_hi, ks, p.H, row_bytes, ks * row_bytes, kBN, 1) ||
        !make_map(&tm_klo, p.k_lo, ks, p.H, row_bytes, ks * row_bytes, kBN, 1) ||
        !make_map(&tm_vhi, p.v_hi, p.H, nk, row_bytes, p.H * row_bytes, 1, kBN) ||
        !make_map(&tm_vlo, p.v_lo, p.H, nk, row_bytes, p.H * row_bytes, 1, kBN))
        return cudaErrorInvalidValue;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(attn_fwd_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kSmemBytes));
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    Params prm;
    prm.q_hat = p.q_hat;
    prm.out = p.out;
    prm.status = status;
    prm.wait_limit = wait_limit;
    prm.q_stride = p.q_stride;
    prm.q_len = p.q_len;
    prm.k_len = p.k_len;
    prm.H = p.H;
    prm.tiles_per_seg = (p.q_len + kBM - 1) / kBM;
    dim3 grid(p.n_seg * prm.tiles_per_seg, p.H);
    attn_fwd_f32_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tm_khi, tm_klo, tm_vhi, tm_vlo, prm);
    return cudaPeekAtLastError();
}

}  // namespace vggt
