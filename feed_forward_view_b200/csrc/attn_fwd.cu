// attn_fwd.cu -- FlashAttention-style forward for sm_100a: softmax(Q K^T / 8) V
// over head dim 64, bf16 in / bf16 out, fp32 scores and accumulators.
//
// ("Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V", Section V slides of the
//  VGGT paper-report deck; frame/global key sets from its "Global + Frame
//  Attention" slide; shapes [B, N, 16, 64] from the vggt-jax README table.)
//
// One CTA owns two 128-row query tiles of one head (256 queries) and streams
// that head's keys/values in 128-row blocks:
//
//   warp 0      TMA producer: Q tiles once, then K_j / V_j into a 3-stage ring.
//   warp 1      MMA issuer (one thread): S_t = Q_t K_j^T (SS, M=128 N=128 K=64)
//               into TMEM, and O_t += P_t V_j (TS: P read from TMEM, M=128
//               N=64 K=128). Allocates / frees the 512 TMEM columns.
//   warps 2-3   idle (they complete the first warpgroup).
//   warps 4-7   softmax for tile 0, warps 8-11 softmax for tile 1: each thread
//               owns one query row (its TMEM lane), reads the row's 128 scores
//               from TMEM, runs the online softmax in fp32 with exp2, writes P
//               as bf16 back to TMEM, and finally normalises O and stores it.
//
// TMEM columns (fp32 unless noted): S0 [0,128) S1 [128,256) O0 [256,320)
// O1 [320,384) P0 [384,448) P1 [448,512) (P: 128 bf16 packed in 64 columns).
//
// Online softmax: m is the running row maximum in log2 units
// (score * log2(e) / 8); p = 2^(score * log2(e)/8 - m). A block whose maximum
// exceeds m by more than kLazy (8, i.e. p <= 256) triggers a rescale of O and
// of the running sum l by 2^(m_old - m_new); smaller increases keep the stale
// m, which is exact because the final O / l uses the same m for both.
//
// Ordering: the MMA thread issues, per key block j and tile t, PV_{t,j-1} and
// then S_{t,j}, and commits S_{t,j} to bar_s[t]. A tcgen05.commit tracks every
// earlier tcgen05 operation of the thread, so when the softmax warps see
// S_{t,j} complete, PV_{t,j-1} has also finished: P_t may be overwritten and
// O_t may be rescaled in place.
//
// Every wait is bounded (vggt::mbar_wait); on timeout the CTA records the
// timeout in the device status word, stops issuing work, drains what it has
// in flight and frees its tensor memory before exiting.
#include <cuda.h>
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "vggt_internal.h"

namespace vggt {
namespace {

constexpr int kBM = 128;                       // query rows per tile
constexpr int kBN = 128;                       // keys per block
constexpr int kStages = 3;                     // K/V ring depth
constexpr int kTileBytes = kBM * kHeadDim * 2; // 16 KB per bf16 tile
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
// TMEM column of S_t, O_t and P_t for query tile t in {0, 1}.
__device__ __forceinline__ constexpr uint32_t col_s(int t) { return 128u * t; }
__device__ __forceinline__ constexpr uint32_t col_o(int t) { return 256u + 64u * t; }
__device__ __forceinline__ constexpr uint32_t col_p(int t) { return 384u + 64u * t; }
constexpr float kScaleLog2 = 0.125f * 1.4426950408889634f;  // log2(e) / sqrt(64)
constexpr float kLazy = 8.0f;

struct SharedStorage {
    uint8_t q[2][kTileBytes];
    uint8_t k[kStages][kTileBytes];
    uint8_t v[kStages][kTileBytes];
    uint64_t bar_q;
    uint64_t bar_kfull[kStages];
    uint64_t bar_kempty[kStages];
    uint64_t bar_vfull[kStages];
    uint64_t bar_vempty[kStages];
    uint64_t bar_s[2];
    uint64_t bar_p[2];
    uint64_t bar_o;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kSmemBytes = sizeof(SharedStorage) + 1024;  // + alignment slack

struct Params {
    uint16_t* out;   // [n_seg*q_len, H, 64]
    int* status;     // device status word
    long long wait_limit;
    int q_len, k_len, H;
    int pairs_per_seg;
};

// Bounded wait that also gives up once this CTA or any other CTA reported a
// timeout; records a timeout of its own.
struct Waiter {
    long long limit;
    volatile int* abort;
    int* status;

    __device__ __forceinline__ bool operator()(uint32_t bar, uint32_t parity) const {
        if (mbar_try_wait(bar, parity)) return true;
        const long long t0 = clock64();
        while (true) {
            if (mbar_try_wait(bar, parity)) return true;
            if (*abort) return false;
            if (*reinterpret_cast<volatile int*>(status)) {
                *abort = 1;
                return false;
            }
            if (clock64() - t0 > limit) {
                *abort = 1;
                atomicOr(status, kStatusTimeout);
                return false;
            }
        }
    }
};

// Wait used while draining on the way out: ignores the abort flags.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, long long limit) {
    if (mbar_try_wait(bar, parity)) return;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) return;
    }
}

// Row maximum of 128 scores with 8 independent running maxima (little extra
// register pressure next to the 128 live scores).
__device__ __forceinline__ float row_max128(const float (&s)[128]) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = s[i];
#pragma unroll
    for (int c = 8; c < 128; ++c) m[c & 7] = fmaxf(m[c & 7], s[c]);
    return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])), fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const Params prm) {
    extern __shared__ uint8_t smem_raw[];
    SharedStorage& sm = *reinterpret_cast<SharedStorage*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int seg = blockIdx.x / prm.pairs_per_seg;
    const int pair = blockIdx.x - seg * prm.pairs_per_seg;
    const int h = blockIdx.y;
    const int n_qtiles = (prm.q_len + kBM - 1) / kBM;
    const int tile0 = 2 * pair;                          // first tile in the segment
    const int ntile = min(2, n_qtiles - tile0);          // 1 or 2
    const int q_row0 = seg * prm.q_len + tile0 * kBM;    // global row of tile 0
    const int k_row0 = seg * prm.k_len;
    const int nkb = (prm.k_len + kBN - 1) / kBN;
    const int last_valid = prm.k_len - (nkb - 1) * kBN;  // keys in the last block

    // Shared-memory addresses of the barriers and tiles; stage / tile indices
    // are runtime values, so they are formed arithmetically (no local arrays).
    const uint32_t bar_q = smem_u32(&sm.bar_q);
    const uint32_t bar_kfull0 = smem_u32(&sm.bar_kfull[0]);
    const uint32_t bar_kempty0 = smem_u32(&sm.bar_kempty[0]);
    const uint32_t bar_vfull0 = smem_u32(&sm.bar_vfull[0]);
    const uint32_t bar_vempty0 = smem_u32(&sm.bar_vempty[0]);
    const uint32_t bar_s0 = smem_u32(&sm.bar_s[0]);
    const uint32_t bar_p0 = smem_u32(&sm.bar_p[0]);
    const uint32_t bar_o = smem_u32(&sm.bar_o);
    const uint32_t q_smem0 = smem_u32(sm.q[0]);
    const uint32_t k_smem0 = smem_u32(sm.k[0]);
    const uint32_t v_smem0 = smem_u32(sm.v[0]);
    auto bar_kfull = [&](int s) { return bar_kfull0 + 8u * s; };
    auto bar_kempty = [&](int s) { return bar_kempty0 + 8u * s; };
    auto bar_vfull = [&](int s) { return bar_vfull0 + 8u * s; };
    auto bar_vempty = [&](int s) { return bar_vempty0 + 8u * s; };
    auto bar_s = [&](int t) { return bar_s0 + 8u * t; };
    auto bar_p = [&](int t) { return bar_p0 + 8u * t; };
    auto q_smem = [&](int t) { return q_smem0 + static_cast<uint32_t>(kTileBytes) * t; };
    auto k_smem = [&](int s) { return k_smem0 + static_cast<uint32_t>(kTileBytes) * s; };
    auto v_smem = [&](int s) { return v_smem0 + static_cast<uint32_t>(kTileBytes) * s; };

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_kfull(s), 1);
            mbar_init(bar_kempty(s), 1);
            mbar_init(bar_vfull(s), 1);
            mbar_init(bar_vempty(s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar_s(t), 1);
            mbar_init(bar_p(t), 4);  // one arrival per softmax warp
        }
        mbar_init(bar_o, 1);
        sm.abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const Waiter wait{prm.wait_limit, &sm.abort, prm.status};

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int n_issued = 0;  // K/V blocks whose loads were started
            mbar_arrive_expect_tx(bar_q, ntile * kTileBytes);
            tma_load_3d(q_smem(0), &tm_q, bar_q, 0, q_row0, h);
            if (ntile == 2) tma_load_3d(q_smem(1), &tm_q, bar_q, 0, q_row0 + kBM, h);
            bool v_pending = false;  // K of the last block started, V not
            for (int j = 0; j < nkb; ++j) {
                const int s = j % kStages;
                const uint32_t use = j / kStages;
                if (use > 0 && !wait(bar_kempty(s), (use - 1) & 1)) break;
                mbar_arrive_expect_tx(bar_kfull(s), kTileBytes);
                tma_load_3d(k_smem(s), &tm_k, bar_kfull(s), 0, k_row0 + j * kBN, h);
                ++n_issued;
                if (use > 0 && !wait(bar_vempty(s), (use - 1) & 1)) {
                    v_pending = true;
                    break;
                }
                mbar_arrive_expect_tx(bar_vfull(s), kTileBytes);
                tma_load_3d(v_smem(s), &tm_v, bar_vfull(s), 0, h, k_row0 + j * kBN);
            }
            // Every copy this CTA started must land before the CTA exits: the
            // last kStages blocks started are the only ones that can still be
            // in flight.
            drain_wait(bar_q, 0, prm.wait_limit);
            for (int j = max(0, n_issued - kStages); j < n_issued; ++j) {
                const int s = j % kStages;
                const uint32_t par = (j / kStages) & 1;
                drain_wait(bar_kfull(s), par, prm.wait_limit);
                if (!(v_pending && j == n_issued - 1)) drain_wait(bar_vfull(s), par, prm.wait_limit);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, kHeadDim, true);
            bool ok = wait(bar_q, 0);
            tc_fence_after();
            for (int j = 0; ok && j <= nkb; ++j) {
                const int s = j % kStages;
                const int sp = (j + kStages - 1) % kStages;  // stage of block j-1
                if (j < nkb && !wait(bar_kfull(s), (j / kStages) & 1)) break;
                if (j > 0 && !wait(bar_vfull(sp), ((j - 1) / kStages) & 1)) break;
                tc_fence_after();
                const uint64_t kdesc = smem_desc_sw128(k_smem(s), 16, 1024);
                const uint64_t vdesc = smem_desc_sw128(v_smem(sp), 16, 1024);
                for (int t = 0; t < ntile; ++t) {
                    if (j > 0) {
                        if (!wait(bar_p(t), (j - 1) & 1)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        // O_t (+)= P_t V_{j-1}: 8 steps of 16 keys.
#pragma unroll
                        for (int kk = 0; kk < kBN / 16; ++kk)
                            mma_ts(tmem + col_o(t), tmem + col_p(t) + kk * 8,
                                   vdesc + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_o,
                                   (j > 1 || kk > 0) ? 1u : 0u);
                    }
                    if (j < nkb) {
                        // S_t = Q_t K_j^T: 4 steps of 16 head dims.
                        const uint64_t qdesc = smem_desc_sw128(q_smem(t), 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < kHeadDim / 16; ++kk)
                            mma_ss(tmem + col_s(t), qdesc + static_cast<uint64_t>((kk * 32) >> 4),
                                   kdesc + static_cast<uint64_t>((kk * 32) >> 4), idesc_s,
                                   kk > 0 ? 1u : 0u);
                        mma_commit(bar_s(t));
                    }
                }
                if (!ok) break;
                if (j < nkb) mma_commit(bar_kempty(s));
                if (j > 0) mma_commit(bar_vempty(sp));
            }
            // Completes once every MMA issued above has finished; the softmax
            // warps wait on it before reading O, and it doubles as the drain.
            mma_commit(bar_o);
            drain_wait(bar_o, 0, prm.wait_limit);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------ softmax
        const int t = (warp >> 2) - 1;
        const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
        const int row = quarter * 32 + lane;
        if (t < ntile) {
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            float m = 0.f, l = 0.f;
            bool ok = true;
            for (int j = 0; j < nkb; ++j) {
                if (!wait(bar_s(t), j & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float s[128];
                {
                    uint32_t r[64];
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        tmem_ld64(lane_base + col_s(t) + 64 * c, r);
#pragma unroll
                        for (int i = 0; i < 64; ++i) s[64 * c + i] = __uint_as_float(r[i]);
                    }
                }
                if (j == nkb - 1 && last_valid < kBN) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c >= last_valid) s[c] = -INFINITY;
                }
                const float mx = row_max128(s) * kScaleLog2;
                // Lazy rescale: only when the block maximum exceeds the running
                // maximum by more than kLazy (log2 units) anywhere in the warp.
                float f = 1.0f;
                bool rescale = false;
                if (j == 0) {
                    m = mx;
                } else {
                    const bool need = mx > m + kLazy;
                    rescale = __any_sync(0xFFFFFFFFu, need);
                    if (need) {
                        f = ex2_approx(m - mx);
                        m = mx;
                    }
                }
                float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                uint32_t pk[64];
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float p0 = ex2_approx(fmaf(s[2 * c], kScaleLog2, -m));
                    const float p1 = ex2_approx(fmaf(s[2 * c + 1], kScaleLog2, -m));
                    part[c & 7] += p0 + p1;
                    pk[c] = pack_bf16x2(p0, p1);
                }
                tmem_st64(lane_base + col_p(t), pk);
                l = l * f + (((part[0] + part[1]) + (part[2] + part[3])) +
                             ((part[4] + part[5]) + (part[6] + part[7])));
                if (rescale) {
                    // O_t holds sum_{i<j} P_i V_i at the old maximum (PV_{t,j-1}
                    // finished before S_{t,j} was signalled).
                    uint32_t o[64];
                    tmem_ld64(lane_base + col_o(t), o);
#pragma unroll
                    for (int i = 0; i < 64; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                    tmem_st64(lane_base + col_o(t), o);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_p(t));
            }
            if (ok && wait(bar_o, 0)) {
                tc_fence_after();
                const int row_in_seg = (tile0 + t) * kBM + row;
                const float inv = 1.0f / l;
                uint32_t o[64];
                tmem_ld64(lane_base + col_o(t), o);
                if (row_in_seg < prm.q_len) {
                    const size_t grow = static_cast<size_t>(seg) * prm.q_len + row_in_seg;
                    uint4* dst = reinterpret_cast<uint4*>(prm.out + (grow * prm.H + h) * kHeadDim);
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(o[8 * v4 + 0]) * inv,
                                          __uint_as_float(o[8 * v4 + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(o[8 * v4 + 2]) * inv,
                                          __uint_as_float(o[8 * v4 + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(o[8 * v4 + 4]) * inv,
                                          __uint_as_float(o[8 * v4 + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(o[8 * v4 + 6]) * inv,
                                          __uint_as_float(o[8 * v4 + 7]) * inv);
                        dst[v4] = w;
                    }
                }
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D bf16 tensor map with a {64, box1, box2} box and 128-byte swizzling.
bool make_map(CUtensorMap* map, const void* base, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
              uint64_t stride2_bytes, uint32_t box1, uint32_t box2) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), d1, d2};
    const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kHeadDim), box1, box2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

__global__ void wait_probe_kernel(int* status, long long limit) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort = 0;
        fence_barrier_init();
        // Nothing ever arrives on `bar`: the wait must run out.
        if (!mbar_wait(smem_u32(&bar), 0, limit, &abort)) atomicOr(status, kStatusTimeout);
    }
}

}  // namespace

cudaError_t launch_attention(const AttnProblem& p, int* status, long long wait_limit,
                             cudaStream_t stream) {
    if (p.n_seg <= 0 || p.H <= 0 || p.q_len <= 0 || p.k_len <= 0) return cudaSuccess;
    const uint64_t nq = static_cast<uint64_t>(p.n_seg) * p.q_len;
    const uint64_t nk = static_cast<uint64_t>(p.n_seg) * p.k_len;
    const uint64_t row_bytes = kHeadDim * 2;
    CUtensorMap tm_q, tm_k, tm_v;
    // q_hat / k_hat: [H][n][64] -> dims {64, n, H}, box {64, 128, 1}
    if (!make_map(&tm_q, p.q_hat, nq, p.H, row_bytes, nq * row_bytes, kBM, 1) ||
        !make_map(&tm_k, p.k_hat, nk, p.H, row_bytes, nk * row_bytes, kBN, 1) ||
        // v: [n][H][64] -> dims {64, H, n}, box {64, 1, 128}
        !make_map(&tm_v, p.v, p.H, nk, row_bytes, p.H * row_bytes, 1, kBN))
        return cudaErrorInvalidValue;

    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kSmemBytes));
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    Params prm;
    prm.out = p.out;
    prm.status = status;
    prm.wait_limit = wait_limit;
    prm.q_len = p.q_len;
    prm.k_len = p.k_len;
    prm.H = p.H;
    const int n_qtiles = (p.q_len + kBM - 1) / kBM;
    prm.pairs_per_seg = (n_qtiles + 1) / 2;
    dim3 grid(p.n_seg * prm.pairs_per_seg, p.H);
    attn_fwd_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tm_q, tm_k, tm_v, prm);
    return cudaPeekAtLastError();
}

cudaError_t launch_wait_probe(int* status, long long wait_limit, cudaStream_t stream) {
    wait_probe_kernel<<<1, 32, 0, stream>>>(status, wait_limit);
    return cudaPeekAtLastError();
}

}  // namespace vggt
