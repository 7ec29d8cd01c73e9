// attn_fwd.cu -- FlashAttention-style forward for sm_100a: softmax(Q K^T / 8) V
// over head dim 64, bf16 in / bf16 out, fp32 scores and accumulators.
//
// ("Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V", Section V slides of the
//  VGGT paper-report deck; frame/global key sets from its "Global + Frame
//  Attention" slide; shapes [B, N, 16, 64] from the vggt-jax README table.)
//
// One CTA owns two 128-row query tiles of one head (256 queries) and streams
// that head's keys/values in 80-row blocks:
//
//   warp 0      TMA producer: Q tiles once, then K_j and V_j together into a
//               5-slot ring (one full / one empty barrier per slot).
//   warps 1, 2  MMA issuers, one per query tile t. The whole warp runs the
//               loop; one elected lane issues the tcgen05 instructions:
//               S_{t,j} = Q_t K_j^T (SS, M=128 N=80 K=64) into TMEM and
//               [O_t | l_t] += P_{t,j} [V_j | 1] (TS: P read from TMEM, M=128
//               N=80 K=80). A tcgen05.mma costs its issuing thread about as
//               long as a small MMA takes to run, so each tile gets an issuer.
//   warp 3      idle (completes the first warpgroup).
//   warps 4-7   softmax for tile 0, warps 8-11 softmax for tile 1: each thread
//               owns one query row (its TMEM lane), reads the row's 80 scores
//               from TMEM, runs the online softmax in fp32 with exp2, writes P
//               as bf16 back to TMEM, and finally normalises O and stores it.
//
// Row sums on the tensor core: the PV MMA's B operand is 80 columns wide --
// V_j (64 columns) followed by a constant shared-memory tile whose first
// column is 1 and the rest 0 (the descriptor's leading byte offset points
// from each V slot to it). Column 64 of the accumulator therefore collects
// l = sum_j P_j from the same bf16 P that multiplies V, and the softmax warps
// do no additions of their own.
//
// TMEM columns, tile t: S_{t,0} [256t, +80), S_{t,1} [256t + 80, +80) (fp32),
// [O_t | l_t] [256t + 160, +80) (fp32); 496 of 512 used. P_{t,b} (80 bf16 per
// row, packed in 40 columns) is written over the first half of S_{t,b} once
// the scores have been read. S is double-buffered: the issuer computes
// S_{t,j+1} while the softmax warps work on block j.
//
// Issue order for tile t: S_{t,0}, S_{t,1}, then for every block j:
// [P_{t,j} ready] PV_{t,j}, commit kv_empty[j's slot], [K_{j+2} loaded]
// S_{t,j+2} into buffer j%2 (after PV_{t,j} has read P_{t,j} from it: the
// tcgen05 MMAs of one thread run in issue order), commit bar_s[t][j%2]; at the
// end, commit bar_o[t]. A commit tracks every earlier tcgen05 operation of the
// thread, so S_{t,j} complete implies PV_{t,j-2} finished (P_{t,j} may be
// written over buffer j%2) and S_{t,j+1} complete implies PV_{t,j-1} finished
// (O_t may be rescaled).
//
// Barrier phases: a parity wait is unambiguous only while the barrier is at
// most one phase away from the awaited one, in either direction. bar_s and
// bar_p exist once per S buffer (blocks b, b+2, ...): the previous phase of
// the same buffer (block j-2) has always been observed, and block j+2 cannot
// start before block j is consumed. The K/V ring follows the same rule.
//
// Online softmax: m is the running row maximum in log2 units
// (score * log2(e) / 8); p = 2^(score * log2(e)/8 - m). A block whose maximum
// exceeds m by more than kLazy (8, i.e. p <= 256) triggers a rescale of
// [O | l] by 2^(m_old - m_new); smaller increases keep the stale m, which is
// exact because the final O / l uses the same m for both. After the QK
// LayerNorm every |score| <= 8 (|q_hat|, |k_hat| <= 8): 2^x is only ever
// needed for x in [-24, 24], so the last block, which has no later S to wait
// on for the rescale, simply keeps the stale maximum (p <= 2^24 stays far
// inside fp32 and bf16 range).
//
// Every wait is bounded; on timeout the CTA records the timeout in the device
// status word, stops issuing work, drains what it has in flight and frees its
// tensor memory before exiting.
#include <cuda.h>
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "vggt_internal.h"

namespace vggt {
namespace {

constexpr int kBM = 128;                          // query rows per tile
constexpr int kBN = 80;                           // keys per block
constexpr int kStages = 5;                        // K/V ring depth
constexpr int kQTileBytes = kBM * kHeadDim * 2;   // 16 KB
constexpr int kKVTileBytes = kBN * kHeadDim * 2;  // 10 KB
constexpr int kOCols = kHeadDim + 16;             // O (64) and the row-sum block (16)
constexpr int kThreads = 384;
// Register split: 168 per thread at launch (the cap for 12 warps); the
// TMA/MMA warpgroup gives up to 80, the two softmax warpgroups take 208:
// 128 * 80 + 256 * 208 = 63488 <= 384 * 168.
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kRegsControl = 80;
constexpr uint32_t kRegsSoftmax = 208;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;

// TMEM column of S_{t,b} (P_{t,b} aliases its first 40 columns) and of
// [O_t | l_t].
__device__ __forceinline__ constexpr uint32_t col_s(int t, int b) { return 256u * t + 80u * b; }
__device__ __forceinline__ constexpr uint32_t col_o(int t) { return 256u * t + 160u; }

constexpr float kScaleLog2 = 0.125f * 1.4426950408889634f;  // log2(e) / sqrt(64)
constexpr float kLazy = 8.0f;

// Exponentials per key block: of every 8 consecutive score pairs,
// kExp2OnFma pairs are evaluated on the FMA pipe (polynomial below) and the
// rest with the MUFU ex2 instruction, so that the two units share the work.
#ifndef VGGT_EXP2_ON_FMA_PER8
#define VGGT_EXP2_ON_FMA_PER8 3
#endif
constexpr int kExp2OnFma = VGGT_EXP2_ON_FMA_PER8;

// 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on [-1/2, 1/2]: minimax in relative error
// (Remez exchange, fit by fit_exp2_poly.py in this directory); worst relative
// error of the whole float32 evaluation over [-24, 8] is 7.5e-5.
constexpr float kExp2C0 = 9.999280572e-01f;
constexpr float kExp2C1 = 6.932609677e-01f;
constexpr float kExp2C2 = 2.426111251e-01f;
constexpr float kExp2C3 = 5.517166853e-02f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

// 2^x on the FMA pipe for x in [-125, 127]: x = j + f with j = round(x)
// (taken by adding 1.5 * 2^23 in round-to-nearest, which leaves j in the low
// mantissa bits of t = x + 1.5 * 2^23) and f = x - j exactly, |f| <= 1/2;
// then 2^x = p(f) * 2^j, with 2^j applied by adding j << 23 to the bit
// pattern of p(f). The attention scores keep x in [-24, 24].
struct SharedStorage {
    uint8_t q[2][kQTileBytes];
    uint8_t kv[kStages][2][kKVTileBytes];  // [slot][K, V]
    uint8_t ones[kKVTileBytes];            // [1, 0, ..., 0] per key row, 128B-swizzled
    uint64_t bar_q;
    uint64_t bar_kvfull[kStages];
    uint64_t bar_kvempty[kStages];
    uint64_t bar_s[2][2];  // [tile][buffer]: S_{t,j} computed (blocks j = b, b+2, ...)
    uint64_t bar_p[2][2];  // [tile][buffer]: P_{t,j} written (blocks j = b, b+2, ...)
    uint64_t bar_o[2];     // [tile]: every MMA of the tile finished (once)
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
// timeout; records a timeout of its own. The barrier is polled back to back
// (try_wait itself suspends the thread for a while); the abort flag, the clock
// and the global status word are only looked at every 256 polls, so that a
// phase that completes is noticed within one poll and not one global-memory
// round trip later.
struct Waiter {
    long long limit;
    volatile int* abort;
    int* status;

    __device__ __forceinline__ bool operator()(uint32_t bar, uint32_t parity) const {
        if (mbar_try_wait(bar, parity)) return true;
        const long long t0 = clock64();
        for (uint32_t it = 1;; ++it) {
            if (mbar_try_wait(bar, parity)) return true;
            if ((it & 255u) == 0) {
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

// Row maximum of 80 scores: 8 independent running maxima fed two scores at a
// time with the three-input max of sm_100.
__device__ __forceinline__ float row_max80(const float (&s)[kBN]) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = s[i];
#pragma unroll
    for (int k = 0; k < 36; ++k) m[k & 7] = fmax3(m[k & 7], s[8 + 2 * k], s[9 + 2 * k]);
    return fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// p = 2^(s * log2(e)/8 - m) for 80 scores, packed to bf16 pairs in pk.
// kMixed: share the exponentials between the FMA pipe and MUFU; otherwise
// MUFU only (blocks with masked -inf scores). Written in phases over all 40
// pairs -- exponents, every MUFU ex2, then each polynomial step for every
// FMA-pipe pair, then the packing -- so that long runs of independent
// instructions hide the latency of each step (the MUFU results are not
// needed until the end).
template <bool kMixed>
__device__ __forceinline__ void exp_pack_row(const float (&s)[kBN], float m, uint32_t (&pk)[kBN / 2]) {
    constexpr int kPairs = kBN / 2;
    const uint64_t scale2 = f2_pack(kScaleLog2, kScaleLog2);
    const uint64_t negm2 = f2_pack(-m, -m);
    auto on_fma = [](int c) { return kMixed && (c & 7) < kExp2OnFma; };
    uint64_t x[kPairs];
#pragma unroll
    for (int c = 0; c < kPairs; ++c) x[c] = f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), scale2, negm2);
    float p[kBN];
#pragma unroll
    for (int c = 0; c < kPairs; ++c)
        if (!on_fma(c)) {
            float x0, x1;
            f2_unpack(x[c], x0, x1);
            p[2 * c] = ex2_approx(x0);
            p[2 * c + 1] = ex2_approx(x1);
        }
    // FMA pipe: x = j + f, 2^x = p(f) * 2^j (see above), one step at a time.
    uint64_t tt[kPairs], ff[kPairs];
#pragma unroll
    for (int c = 0; c < kPairs; ++c)
        if (on_fma(c)) tt[c] = f2_add(x[c], f2_pack(kRoundMagic, kRoundMagic));
#pragma unroll
    for (int c = 0; c < kPairs; ++c)
        if (on_fma(c)) ff[c] = f2_add(tt[c], f2_pack(-kRoundMagic, -kRoundMagic));
#pragma unroll
    for (int c = 0; c < kPairs; ++c)
        if (on_fma(c)) ff[c] = f2_fma(ff[c], f2_pack(-1.0f, -1.0f), x[c]);
#pragma unroll
    for (int c = 0; c < kPairs; ++c)
        if (on_fma(c)) x[c] = f2_fma(f2_pack(kExp2C3, kExp2C3), ff[c], f2_pack(kExp2C2, kExp2C2));
#pragma unroll
    for (int c = 0; c < kPairs; ++c)
        if (on_fma(c)) x[c] = f2_fma(x[c], ff[c], f2_pack(kExp2C1, kExp2C1));
#pragma unroll
    for (int c = 0; c < kPairs; ++c)
        if (on_fma(c)) x[c] = f2_fma(x[c], ff[c], f2_pack(kExp2C0, kExp2C0));
#pragma unroll
    for (int c = 0; c < kPairs; ++c)
        if (on_fma(c)) {
            uint32_t q0, q1, t0, t1;
            u2_unpack(x[c], q0, q1);
            u2_unpack(tt[c], t0, t1);
            p[2 * c] = __uint_as_float(q0 + (t0 << 23));
            p[2 * c + 1] = __uint_as_float(q1 + (t1 << 23));
        }
#pragma unroll
    for (int c = 0; c < kPairs; ++c) pk[c] = pack_bf16x2(p[2 * c], p[2 * c + 1]);
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

    // Shared-memory addresses of the barriers and tiles; slot / tile indices
    // are runtime values, so they are formed arithmetically (no local arrays).
    const uint32_t bar_q = smem_u32(&sm.bar_q);
    const uint32_t bar_kvfull0 = smem_u32(&sm.bar_kvfull[0]);
    const uint32_t bar_kvempty0 = smem_u32(&sm.bar_kvempty[0]);
    const uint32_t bar_s0 = smem_u32(&sm.bar_s[0][0]);
    const uint32_t bar_p0 = smem_u32(&sm.bar_p[0][0]);
    const uint32_t bar_o0 = smem_u32(&sm.bar_o[0]);
    const uint32_t q_smem0 = smem_u32(sm.q[0]);
    const uint32_t kv_smem0 = smem_u32(sm.kv[0][0]);
    const uint32_t ones_smem = smem_u32(sm.ones);
    auto bar_kvfull = [&](int s) { return bar_kvfull0 + 8u * s; };
    auto bar_kvempty = [&](int s) { return bar_kvempty0 + 8u * s; };
    auto bar_s = [&](int t, int b) { return bar_s0 + 16u * t + 8u * b; };
    auto bar_p = [&](int t, int b) { return bar_p0 + 16u * t + 8u * b; };
    auto bar_o = [&](int t) { return bar_o0 + 8u * t; };
    auto q_smem = [&](int t) { return q_smem0 + static_cast<uint32_t>(kQTileBytes) * t; };
    auto k_smem = [&](int s) { return kv_smem0 + static_cast<uint32_t>(2 * kKVTileBytes) * s; };
    auto v_smem = [&](int s) { return k_smem(s) + static_cast<uint32_t>(kKVTileBytes); };

    // The constant [1, 0, ..., 0] rows in the 128-byte-swizzled layout the
    // MMA reads: the 16-byte chunk c of row r sits at chunk c ^ (r % 8), so
    // element 0 of row r lies at byte r * 128 + (r % 8) * 16.
    for (int i = threadIdx.x; i < kKVTileBytes / 16; i += kThreads) {
        const int r = i >> 3, chunk = i & 7;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (chunk == (r & 7)) w.x = 0x3F80u;  // bf16 1.0 in the low half
        reinterpret_cast<uint4*>(sm.ones)[i] = w;
    }
    fence_proxy_async_smem();  // make the generic-proxy writes visible to the MMA

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_kvfull(s), 1);
            mbar_init(bar_kvempty(s), ntile);  // one commit per tile issuer
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar_s(t, 0), 1);
            mbar_init(bar_s(t, 1), 1);
            mbar_init(bar_p(t, 0), 4);  // one arrival per softmax warp
            mbar_init(bar_p(t, 1), 4);
            mbar_init(bar_o(t), 1);
        }
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

    if (warp < 4) regs_dec<kRegsControl>();
    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int n_issued = 0;  // blocks whose loads were started
            mbar_arrive_expect_tx(bar_q, ntile * kQTileBytes);
            tma_load_3d(q_smem(0), &tm_q, bar_q, 0, q_row0, h);
            if (ntile == 2) tma_load_3d(q_smem(1), &tm_q, bar_q, 0, q_row0 + kBM, h);
            for (int j = 0; j < nkb; ++j) {
                const int s = j % kStages;
                const uint32_t use = j / kStages;
                if (use > 0 && !wait(bar_kvempty(s), (use - 1) & 1)) break;
                mbar_arrive_expect_tx(bar_kvfull(s), 2 * kKVTileBytes);
                tma_load_3d(k_smem(s), &tm_k, bar_kvfull(s), 0, k_row0 + j * kBN, h);
                tma_load_3d(v_smem(s), &tm_v, bar_kvfull(s), 0, h, k_row0 + j * kBN);
                ++n_issued;
            }
            // Every copy this CTA started must land before the CTA exits: the
            // last kStages blocks started are the only ones that can still be
            // in flight.
            drain_wait(bar_q, 0, prm.wait_limit);
            for (int j = max(0, n_issued - kStages); j < n_issued; ++j)
                drain_wait(bar_kvfull(j % kStages), (j / kStages) & 1, prm.wait_limit);
        }
    } else if (warp == 1 || warp == 2) {
        // ------------------------------------------------------ MMA issuers
        // The whole warp runs the loop (so the descriptor arithmetic is
        // warp-uniform); every lane polls the barriers and the verdict is
        // made uniform with a vote; one elected lane issues the tcgen05
        // instructions and their commits.
        const int t = warp - 1;
        if (t < ntile) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, kOCols, true);
            const uint64_t qdesc = smem_desc_sw128(q_smem(t), 16, 1024);
            auto uwait = [&](uint32_t bar, uint32_t parity) {
                return __all_sync(0xFFFFFFFFu, wait(bar, parity)) != 0;
            };
            // S_{t,j} = Q_t K_j^T into buffer j % 2: 4 steps of 16 head dims.
            auto issue_s = [&](int j) {
                const uint64_t kdesc = smem_desc_sw128(k_smem(j % kStages), 16, 1024);
                const uint32_t d = tmem + col_s(t, j & 1);
                const uint32_t done = bar_s(t, j & 1);
                if (elect_one()) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kHeadDim / 16; ++kk)
                        mma_ss(d, qdesc + static_cast<uint64_t>((kk * 32) >> 4),
                               kdesc + static_cast<uint64_t>((kk * 32) >> 4), idesc_s, kk > 0 ? 1u : 0u);
                    mma_commit(done);
                }
                __syncwarp();
            };
            bool ok = uwait(bar_q, 0);
            for (int j = 0; ok && j < min(2, nkb); ++j) {
                if (!uwait(bar_kvfull(j % kStages), (j / kStages) & 1)) {
                    ok = false;
                    break;
                }
                issue_s(j);
            }
            for (int j = 0; ok && j < nkb; ++j) {
                const int s = j % kStages;
                if (!uwait(bar_p(t, j & 1), (j >> 1) & 1)) break;
                // [O_t | l_t] (+)= P_{t,j} [V_j | 1]: 5 steps of 16 keys; P sits
                // in the first 40 columns of S_{t, j%2}. The B operand's second
                // 64-column block (the ones tile) lies a leading byte offset
                // away from the V slot.
                const uint32_t vaddr = v_smem(s);
                const uint64_t vdesc = smem_desc_sw128(vaddr, ones_smem - vaddr, 1024);
                const uint32_t a = tmem + col_s(t, j & 1);
                const uint32_t d = tmem + col_o(t);
                const uint32_t first = j > 0 ? 1u : 0u;
                const uint32_t empty = bar_kvempty(s);
                if (elect_one()) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; ++kk)
                        mma_ts(d, a + kk * 8, vdesc + static_cast<uint64_t>((kk * 16 * 128) >> 4),
                               idesc_o, kk > 0 ? 1u : first);
                    mma_commit(empty);  // K_j and V_j no longer needed by this tile
                }
                __syncwarp();
                const int jn = j + 2;
                if (jn < nkb) {
                    if (!uwait(bar_kvfull(jn % kStages), (jn / kStages) & 1)) break;
                    issue_s(jn);
                }
            }
            // Completes once every MMA of this tile has finished: the softmax
            // warps wait on it before the epilogue; it doubles as the drain.
            if (elect_one()) mma_commit(bar_o(t));
            __syncwarp();
            drain_wait(bar_o(t), 0, prm.wait_limit);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------ softmax
        regs_inc<kRegsSoftmax>();
        const int t = (warp >> 2) - 1;
        const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
        const int row = quarter * 32 + lane;
        if (t < ntile) {
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            float m = 0.f;
            bool ok = true;
            for (int j = 0; j < nkb; ++j) {
                const int b = j & 1;
                if (!wait(bar_s(t, b), (j >> 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float s[kBN];
                {
                    uint32_t r[kBN];
                    tmem_ld80(lane_base + col_s(t, b), r);
#pragma unroll
                    for (int i = 0; i < kBN; ++i) s[i] = __uint_as_float(r[i]);
                }
                const bool masked = (j == nkb - 1) && last_valid < kBN;
                if (masked) {
#pragma unroll
                    for (int c = 0; c < kBN; ++c)
                        if (c >= last_valid) s[c] = -INFINITY;
                }
                const float mx = row_max80(s) * kScaleLog2;
                // Lazy rescale: only when the block maximum exceeds the running
                // maximum by more than kLazy (log2 units) anywhere in the warp,
                // and never on the last block (see the header comment).
                float f = 1.0f;
                bool rescale = false;
                if (j == 0) {
                    m = mx;
                } else if (j + 1 < nkb) {
                    const bool need = mx > m + kLazy;
                    rescale = __any_sync(0xFFFFFFFFu, need);
                    if (need) {
                        f = ex2_approx(m - mx);
                        m = mx;
                    }
                }
                uint32_t pk[kBN / 2];
                if (masked)
                    exp_pack_row<false>(s, m, pk);
                else
                    exp_pack_row<true>(s, m, pk);
                tmem_st40(lane_base + col_s(t, b), pk);
                if (rescale) {
                    // [O_t | l_t] must hold sum_{i<j} P_i [V_i | 1]: S_{t,j+1}
                    // complete implies PV_{t,j-1} finished.
                    if (!wait(bar_s(t, b ^ 1), ((j + 1) >> 1) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint32_t o[kOCols];
                    tmem_ld80(lane_base + col_o(t), o);
#pragma unroll
                    for (int i = 0; i < kOCols; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                    tmem_st80(lane_base + col_o(t), o);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_p(t, b));
            }
            if (ok && wait(bar_o(t), 0)) {
                tc_fence_after();
                const int row_in_seg = (tile0 + t) * kBM + row;
                uint32_t o[kOCols];
                tmem_ld80(lane_base + col_o(t), o);
                const float inv = 1.0f / __uint_as_float(o[kHeadDim]);  // l = column 64
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
    // q_hat / k_hat: [H][n][64] -> dims {64, n, H}, box {64, rows, 1}
    if (!make_map(&tm_q, p.q_hat, nq, p.H, row_bytes, nq * row_bytes, kBM, 1) ||
        !make_map(&tm_k, p.k_hat, nk, p.H, row_bytes, nk * row_bytes, kBN, 1) ||
        // v: [n][H][64] -> dims {64, H, n}, box {64, 1, rows}
        !make_map(&tm_v, p.v, p.H, nk, row_bytes, p.H * row_bytes, 1, kBN))
        return cudaErrorInvalidValue;

    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        // The register split (setmaxnreg) needs the full launch allocation
        // (kLaunchRegs per thread); with fewer registers the softmax
        // warpgroups' increase could never be granted. Refuse to launch such
        // a build.
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, attn_fwd_kernel);
        if (e != cudaSuccess) return e;
        if (static_cast<uint32_t>(fa.numRegs) * kThreads < 128 * kRegsControl + 256 * kRegsSoftmax)
            return cudaErrorInvalidConfiguration;
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
