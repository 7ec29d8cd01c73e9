// attn_fwd_f32.cu -- the fp32 mode of the attention: softmax(Q K^T / 8) V with
// fp32 q_hat, k, v in and fp32 out, to about fp32 accuracy, on the bf16
// tensor cores.
//
// ("Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V", Section V slides of the
//  VGGT paper-report deck. The fp32 mode answers the vggt-jax README's
//  precision study: its attention runs in FP32 -- TF32x3 Triton kernels -- for
//  parity with the FP32 reference.)
//
// Every fp32 operand x is carried as kTerms bf16 terms x_0 = bf16(x),
// x_1 = bf16(x - x_0) (and x_2 = bf16(x - x_0 - x_1)). A product a b is the
// sum of the term products a_i b_j with i + j < kTerms -- each a bf16 MMA with
// fp32 accumulation; the dropped ones are typically ~2^-18 (two terms) or
// ~2^-27 (three terms) of a b, at most 2^-16 and 2^-23:
//   two terms:   3 products (0,0) (0,1) (1,0)                    ~2^-17
//   three terms: 6 products (0,0) (0,1) (1,0) (0,2) (1,1) (2,0)   ~fp32
//   S     = sum Q_i K_j^T                  (4 K-steps each, N = 96)
//   [O|l] += sum P_i [V_j | 1 if j == 0]   (6 K-steps each, N = 80 or 64)
// The row sum l comes from the ones column of the products with V_0 (their P
// terms are all of P's terms, so l = sum of P, the P that multiplies V). The
// exponentials must be good to ~2^-22: every one is MUFU ex2. (Sending 2 of
// every 8 score pairs to a degree-5 polynomial on the FMA pipe, as the bf16
// kernel does with degree 3, measured 1.4% slower here: with three or six
// products per useful one the tensor pipe, not MUFU, is the busiest unit.)
//
// The same kernel serves bf16 calls whose QK LayerNorm affine makes the
// scores too large for a bf16 q_hat / k_hat to resolve (an element's
// rounding, 2^-9 of it, moves a score by about 2^-9 |q_hat| |k_hat| / 8; with
// weights of 8 that is several units): Q and K in two terms, as above, but P
// and V in one (the bf16 v itself), the bf16 output of O / l, and the online
// softmax (kTQ = 2, kTP = 1).
//
// One CTA per 128-row query tile of one head. Warps: 0 TMA producer for the
// K terms of a key block (96 keys; 64 in the precise instance, see Cfg), 2
// for the V terms (separate rings: 4 + 4 slots for two terms, 3 + 2 for
// three, 3 + 4 in the precise instance), 1 MMA issuer, 3 idle, 4-11 softmax
// (2 per TMEM lane quarter, half the block's score columns each). Tensor
// memory: the Q terms (32 columns each), S (one column per key), the P terms
// (half that each), [O | l] (80) and its folded sum (80, see kFold). The softmax warps and the issuer meet once
// per key block exactly as in the bf16 kernel (attn_fwd.cu): right after
// loading S_j the softmax warps arrive on bar_c (P_{j-1} written, S free; the
// first warp has checked that K_{j+1} landed), and on that signal the issuer
// issues PV_{j-1} and S_{j+1}. No row maximum either: the prologue bounds
// every score to [-8, 8] (see attn_fwd.cu). The kOnline instance, for a QK
// LayerNorm affine without that bound, keeps a running row maximum exactly as
// the bf16 kernel's online instance does (the two warps of a row swap their
// block maxima through shared memory; the reference moves only when a block's
// maximum exceeds it by more than 8 in log2 units); a move rescales the
// current [O | l] run and, once it holds something, the folded sum.
//
// Every wait is bounded; on timeout the CTA records it in the device status
// word, stops issuing, drains what it has in flight and frees its tensor
// memory.
#include <atomic>

#include <cuda_bf16.h>

#include "attn_common.cuh"

namespace vggt {
namespace {

using attn::drain_wait;
using attn::make_map;
using attn::Waiter;

constexpr int kBM = 128;                          // query rows per CTA
constexpr int kOCols = kHeadDim + 16;             // O (64) and the row-sum block
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 128 + 32 * kSoftmaxWarps;  // 384

// Per term counts -- kTQ for Q and K (the score product), kTP for P and V
// (the value product): the K and V ring depths (separate rings, each with its
// own producer warp, so that a slot of either frees on its own MMA) and the
// tensor memory columns.
//   fp32 mode, two terms (kTQ = kTP = 2): 4 + 4 slots of 2 tiles;
//   three terms (3, 3): 3 + 2 slots of 3 tiles (a third V slot does not fit
//   beside them in 227 KB);
//   precise scores for bf16 calls (2, 1): 64-key blocks, 3 K slots of 2
//   tiles, 4 V slots of one tile (the bf16 v itself); P in one bf16 term and
//   a bf16 output, so the value product needs no fold. With 64 keys a block,
//   a CTA needs 240 of 256 TMEM columns and ~90 KB of shared memory, so two
//   CTAs share an SM (one alone left the SM latency-bound: tensor pipe 48 %,
//   MUFU 47 %, 8 softmax warps).
template <int kTQ, int kTP>
struct Cfg {
    static_assert((kTQ == 2 || kTQ == 3) && (kTP == kTQ || (kTQ == 2 && kTP == 1)), "term counts");
    static constexpr int kBN = kTP == 1 ? 64 : 96;             // keys per block
    static constexpr int kTileBytes = kBN * kHeadDim * 2;      // one kBN x 64 bf16 tile
    static constexpr int kCols = kBN / 2;                      // score columns per softmax thread
    static constexpr int kMinBlocks = kTP == 1 ? 2 : 1;        // resident CTAs per SM
    static constexpr uint32_t kTmemCols = kTP == 1 ? 256 : 512;
    static constexpr int kStagesK = kTP == 1 ? 3 : (kTQ == 2 ? 4 : 3);
    static constexpr int kStagesV = kTP == 1 ? 4 : (kTP == 2 ? 4 : 2);
    static constexpr int kPairsS = kTQ * (kTQ + 1) / 2;   // term products kept in S
    static constexpr int kPairsPV = kTP * (kTP + 1) / 2;  // and in [O | l]
    static constexpr bool kFoldOn = kTP > 1;              // fp32 outputs: fold every kFold blocks
    static constexpr bool kBf16Out = kTP == 1;
    static constexpr uint32_t kColQ = 0;                  // 32 per term
    static constexpr uint32_t kColS = 32 * kTQ;
    static constexpr uint32_t kColP = kColS + kBN;        // kBN / 2 per term
    static constexpr uint32_t kColO = kColP + (kBN / 2) * kTP;
    static constexpr uint32_t kColA = kColO + kOCols;     // the folded partial sums
    static_assert((kFoldOn ? kColA : kColO) + kOCols <= kTmemCols, "tensor memory columns");
    static_assert(kCols == 32 || kCols == 48, "score columns per thread");
};

// TMEM loads and stores of the widths the two block sizes use.
template <int N>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 32 || N == 48, "unsupported width");
    if constexpr (N == 32) tmem_ld32(taddr, r);
    if constexpr (N == 48) tmem_ld48(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_store_cols(uint32_t taddr, const uint32_t (&r)[N]) {
    static_assert(N == 16 || N == 24, "unsupported width");
    if constexpr (N == 16) tmem_st16(taddr, r);
    if constexpr (N == 24) tmem_st24(taddr, r);
}

// The kept term products in order of size: (0,0), then (0,1) (1,0), then
// (0,2) (1,1) (2,0). Product i multiplies term pair_a(i) of the left operand
// with term pair_b(i) of the right one.
__host__ __device__ constexpr int pair_level(int i) { return i == 0 ? 0 : (i < 3 ? 1 : 2); }
__host__ __device__ constexpr int pair_a(int i) { return i - pair_level(i) * (pair_level(i) + 1) / 2; }
__host__ __device__ constexpr int pair_b(int i) { return pair_level(i) - pair_a(i); }
static_assert(pair_a(2) == 1 && pair_b(2) == 0 && pair_a(3) == 0 && pair_b(3) == 2 && pair_a(5) == 2 &&
                  pair_b(5) == 0,
              "term pairs");

constexpr float kScaleLog2 = 0.125f * 1.4426950408889634f;  // log2(e) / sqrt(64)

// [O | l] accumulates in tensor memory over kFold key blocks at a time; the
// softmax warps then fold that partial into a second tensor-memory sum with
// round-to-nearest fp32 adds, and the next block's products start afresh.
// Accumulating all 385 blocks of a 36 909-key row in place lost ~1e-4
// relative (measured: the tensor core's accumulator adds do not round to
// nearest, and their error grows with the number of updates, so three terms
// came out worse than two); folding every 8 blocks caps each run of in-place
// updates.
constexpr int kFold = 8;

// 8 consecutive columns at each of two addresses, waited for.
__device__ __forceinline__ void tmem_ld8x2(uint32_t taddr0, uint32_t taddr1, uint32_t (&r0)[8], uint32_t (&r1)[8]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%16];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%8, %9, %10, %11, %12, %13, %14, %15}, [%17];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r0[0]), "=r"(r0[1]), "=r"(r0[2]), "=r"(r0[3]), "=r"(r0[4]), "=r"(r0[5]), "=r"(r0[6]), "=r"(r0[7]),
          "=r"(r1[0]), "=r"(r1[1]), "=r"(r1[2]), "=r"(r1[3]), "=r"(r1[4]), "=r"(r1[5]), "=r"(r1[6]), "=r"(r1[7])
        : "r"(taddr0), "r"(taddr1)
        : "memory");
}
// 8 consecutive columns, waited for.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n\t"
        "tcgen05.wait::st.sync.aligned;"
        :
        : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
}

template <int kTQ, int kTP>
struct SharedStorage {
    using C = Cfg<kTQ, kTP>;
    uint8_t k[C::kStagesK][kTQ][C::kTileBytes];  // K terms, 128B-swizzled
    uint8_t v[C::kStagesV][kTP][C::kTileBytes];  // V terms, 128B-swizzled
    uint8_t ones[C::kTileBytes];                 // [1, 0, ..., 0] per key row, 128B-swizzled
    uint64_t bar_kfull[C::kStagesK];
    uint64_t bar_kempty[C::kStagesK];
    uint64_t bar_vfull[C::kStagesV];
    uint64_t bar_vempty[C::kStagesV];
    uint64_t bar_q;      // the Q terms in tensor memory
    uint64_t bar_s;      // S_j computed
    uint64_t bar_c;      // P_{j-1} written and S_j read
    uint64_t bar_pfree;  // PV_j finished
    uint64_t bar_o;      // every MMA finished (once)
    uint32_t tmem_base;
    int abort;
};
// Online instance only, placed after SharedStorage: per lane quarter the pair
// barrier of its two softmax warps and their block maxima, double buffered by
// block parity ([quarter][parity][half][lane]).
struct OnlineShared {
    uint64_t bar_pair[4];
    float xchg[4][2][2][32];
};
constexpr float kRescaleLog2 = 8.0f;  // see attn_fwd.cu

template <int kTQ, int kTP, bool kOnline>
constexpr size_t smem_bytes() {
    return sizeof(SharedStorage<kTQ, kTP>) + (kOnline ? sizeof(OnlineShared) : 0) + 1024;  // + alignment slack
}
static_assert(smem_bytes<2, 2, true>() <= 227 * 1024 && smem_bytes<3, 3, true>() <= 227 * 1024 &&
                  smem_bytes<2, 1, true>() <= 227 * 1024,
              "shared memory beyond the per-CTA limit");
// two (2, 1) CTAs per SM: 228 KB per SM, 1 KB of it reserved per CTA
static_assert(2 * (smem_bytes<2, 1, true>() + 1024) <= 228 * 1024, "two precise-mode CTAs do not fit an SM");

// The TMA maps of the K terms (head-major planes) and the V terms
// (token-major), unused entries zero.
struct Maps {
    CUtensorMap k[3];
    CUtensorMap v[3];
};

struct Params {
    const float* q_hat;  // fp32, head planes q_stride rows apart
    void* out;           // [n_seg*q_len, H, 64], fp32 (or bf16 when kTP == 1)
    int* status;
    long long wait_limit;
    long long q_stride;
    int q_len, k_len, H;
    int tiles_per_seg;
    RowMap out_map;      // query row r is stored at output row map_row(out_map, r)
};

// The kTerms bf16 terms of two fp32 values, each packed low half first: one
// paired round-to-nearest conversion per term, the rounded values read back
// from the packed word by bit operations, the remainders exact in fp32.
template <int kTerms>
__device__ __forceinline__ void split_terms(float a, float b, uint32_t (&w)[kTerms]) {
#pragma unroll
    for (int i = 0; i < kTerms; ++i) {
        w[i] = pack_bf16x2(a, b);
        if (i + 1 < kTerms) {
            a -= __uint_as_float(w[i] << 16);
            b -= __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
}

template <int kTQ, int kTP, bool kOnline>
__global__ void __launch_bounds__(kThreads, Cfg<kTQ, kTP>::kMinBlocks)
attn_fwd_f32_kernel(const __grid_constant__ Maps maps, const Params prm) {
    griddep_launch_dependents();
    griddep_wait();  // before any global memory access (pdl.cuh)
    using C = Cfg<kTQ, kTP>;
    constexpr int kBN = C::kBN;
    constexpr int kTileBytes = C::kTileBytes;
    constexpr int kCols = C::kCols;
    constexpr int kSK = C::kStagesK, kSV = C::kStagesV;
    extern __shared__ uint8_t smem_raw[];
    SharedStorage<kTQ, kTP>& sm = *reinterpret_cast<SharedStorage<kTQ, kTP>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    OnlineShared& on = *reinterpret_cast<OnlineShared*>(&sm + 1);  // online instance only

    const int warp = __shfl_sync(0xFFFFFFFFu, static_cast<int>(threadIdx.x >> 5), 0);
    const int lane = threadIdx.x & 31;
    const int seg = blockIdx.x / prm.tiles_per_seg;
    const int tile = blockIdx.x - seg * prm.tiles_per_seg;
    const int h = blockIdx.y;
    const int k_row0 = seg * prm.k_len;
    const int nkb = (prm.k_len + kBN - 1) / kBN;
    const int last_valid = prm.k_len - (nkb - 1) * kBN;

    const uint32_t bar_kfull0 = smem_u32(&sm.bar_kfull[0]);
    const uint32_t bar_kempty0 = smem_u32(&sm.bar_kempty[0]);
    const uint32_t bar_vfull0 = smem_u32(&sm.bar_vfull[0]);
    const uint32_t bar_vempty0 = smem_u32(&sm.bar_vempty[0]);
    const uint32_t bar_q = smem_u32(&sm.bar_q);
    const uint32_t bar_s = smem_u32(&sm.bar_s);
    const uint32_t bar_c = smem_u32(&sm.bar_c);
    const uint32_t bar_pfree = smem_u32(&sm.bar_pfree);
    const uint32_t bar_o = smem_u32(&sm.bar_o);
    const uint32_t k_smem0 = smem_u32(sm.k[0][0]);
    const uint32_t v_smem0 = smem_u32(sm.v[0][0]);
    const uint32_t ones_smem = smem_u32(sm.ones);
    auto bar_kfull = [&](int s) { return bar_kfull0 + 8u * s; };
    auto bar_kempty = [&](int s) { return bar_kempty0 + 8u * s; };
    auto bar_vfull = [&](int s) { return bar_vfull0 + 8u * s; };
    auto bar_vempty = [&](int s) { return bar_vempty0 + 8u * s; };
    auto k_tile = [&](int s, int t) { return k_smem0 + static_cast<uint32_t>(kTileBytes) * (kTQ * s + t); };
    auto v_tile = [&](int s, int t) { return v_smem0 + static_cast<uint32_t>(kTileBytes) * (kTP * s + t); };

    attn::fill_ones_tile(sm.ones, kTileBytes, kThreads);
    fence_proxy_async_smem();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSK; ++s) {
            mbar_init(bar_kfull(s), 1);
            mbar_init(bar_kempty(s), 1);
        }
        for (int s = 0; s < kSV; ++s) {
            mbar_init(bar_vfull(s), 1);
            mbar_init(bar_vempty(s), 1);
        }
        mbar_init(bar_q, kSoftmaxWarps);
        mbar_init(bar_s, 1);
        mbar_init(bar_c, kSoftmaxWarps);
        mbar_init(bar_pfree, 1);
        mbar_init(bar_o, 1);
        if constexpr (kOnline) {
            for (int qr = 0; qr < 4; ++qr) mbar_init(smem_u32(&on.bar_pair[qr]), 2);
        }
        sm.abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if ((warp == 0 || warp == 2) && lane == 0) {
        for (int t = 0; t < (warp == 0 ? kTQ : kTP); ++t) tma_prefetch_desc(warp == 0 ? &maps.k[t] : &maps.v[t]);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = __shfl_sync(0xFFFFFFFFu, sm.tmem_base, 0);
    const Waiter wait{prm.wait_limit, &sm.abort, prm.status};

    if (warp == 0 || warp == 2) {
        // ------------------------------------------ TMA producers: 0 K, 2 V
        if (lane == 0) {
            const bool is_k = warp == 0;
            const int n_st = is_k ? kSK : kSV;
            int n_issued = 0;
            for (int j = 0; j < nkb; ++j) {
                const int s = j % n_st;
                const uint32_t use = j / n_st;
                const uint32_t full = is_k ? bar_kfull(s) : bar_vfull(s);
                if (use > 0 && !wait(is_k ? bar_kempty(s) : bar_vempty(s), (use - 1) & 1)) break;
                mbar_arrive_expect_tx(full, (is_k ? kTQ : kTP) * kTileBytes);
                const int row = k_row0 + j * kBN;
                if (is_k) {
#pragma unroll
                    for (int t = 0; t < kTQ; ++t) tma_load_3d(k_tile(s, t), &maps.k[t], full, 0, row, h);
                } else {
#pragma unroll
                    for (int t = 0; t < kTP; ++t) tma_load_3d(v_tile(s, t), &maps.v[t], full, 0, h, row);
                }
                ++n_issued;
            }
            for (int j = max(0, n_issued - n_st); j < n_issued; ++j)
                drain_wait(is_k ? bar_kfull(j % n_st) : bar_vfull(j % n_st), (j / n_st) & 1, prm.wait_limit);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, false);
        constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, kOCols, true);
        constexpr uint32_t idesc_o64 = idesc_bf16_f32(kBM, kHeadDim, true);
        auto uwait = [&](uint32_t bar, uint32_t parity) {
            return __all_sync(0xFFFFFFFFu, wait(bar, parity)) != 0;
        };
        const uint32_t s_tm = tmem + C::kColS, o_tm = tmem + C::kColO;
        const uint32_t q_tm = tmem + C::kColQ, p_tm = tmem + C::kColP;
        // S_j: the kept products Q_a K_b^T, 4 steps of 16 head dims each (8
        // TMEM columns of Q, 32 bytes of each 128-byte K row)
        auto issue_s = [&](int j) {
            const int s = j % kSK;
            if (elect_one()) {
                tc_fence_after();
#pragma unroll
                for (int i = 0; i < C::kPairsS; ++i) {
                    const uint64_t kd = smem_desc_sw128(k_tile(s, pair_b(i)), 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(s_tm, q_tm + 32 * pair_a(i) + 8 * kk, kd + static_cast<uint64_t>((kk * 32) >> 4),
                               idesc_s, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar_s);
                mma_commit(bar_kempty(s));
            }
            __syncwarp();
        };
        // PV_j: the kept products P_a [V_b | 1], kBN / 16 steps of 16 keys each; the
        // products with V_0 carry the ones column (the B operand's second
        // 64-column block, a leading byte offset away from the V_0 tile), so
        // the row sum collects every term of P
        auto issue_pv = [&](int j) {
            const int s = j % kSV;
            const uint32_t v0_addr = v_tile(s, 0);
            if (elect_one()) {
                tc_fence_after();
#pragma unroll
                for (int i = 0; i < C::kPairsPV; ++i) {
                    const int b = pair_b(i);
                    const uint64_t vd = b == 0 ? smem_desc_sw128(v0_addr, ones_smem - v0_addr, 1024)
                                               : smem_desc_sw128(v_tile(s, b), 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; ++kk)
                        mma_ts(o_tm, p_tm + (kBN / 2) * pair_a(i) + 8 * kk, vd + static_cast<uint64_t>((kk * 16 * 128) >> 4),
                               b == 0 ? idesc_o : idesc_o64,
                               ((C::kFoldOn ? j % kFold != 0 : j > 0) || i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar_pfree);
                mma_commit(bar_vempty(s));
            }
            __syncwarp();
        };
        bool ok = uwait(bar_q, 0) && uwait(bar_kfull(0), 0);
        if (ok) issue_s(0);
        ok = ok && uwait(bar_c, 0);  // S_0 read (and K_1 landed)
        if (ok && nkb > 1) issue_s(1);
        for (int j = 0; ok && j < nkb; ++j) {
            if (!uwait(bar_c, (j + 1) & 1)) break;  // P_j written, S_{j+1} read, K_{j+2} landed
            if (!uwait(bar_vfull(j % kSV), (j / kSV) & 1)) break;
            issue_pv(j);
            if (j + 2 < nkb) issue_s(j + 2);
        }
        if (elect_one()) mma_commit(bar_o);
        __syncwarp();
        drain_wait(bar_o, 0, prm.wait_limit);
    } else if (warp >= 4) {
        // ------------------------------------------------------ softmax
        const int half = (warp - 4) >> 2;  // score columns [kCols*half, +kCols)
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
        // log2(e)/8 in fp32, as kTQ bf16 terms (16 columns each).
        {
            uint32_t qt[kTQ][16];
            if (row_live) {
                const float4* src = reinterpret_cast<const float4*>(
                    prm.q_hat + (static_cast<long long>(h) * prm.q_stride + grow) * kHeadDim + 32 * half);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 w = __ldg(src + i);
                    uint32_t a[kTQ], b[kTQ];
                    split_terms<kTQ>(w.x * kScaleLog2, w.y * kScaleLog2, a);
                    split_terms<kTQ>(w.z * kScaleLog2, w.w * kScaleLog2, b);
#pragma unroll
                    for (int t = 0; t < kTQ; ++t) {
                        qt[t][2 * i] = a[t];
                        qt[t][2 * i + 1] = b[t];
                    }
                }
            } else {
#pragma unroll
                for (int t = 0; t < kTQ; ++t)
#pragma unroll
                    for (int i = 0; i < 16; ++i) qt[t][i] = 0u;
            }
#pragma unroll
            for (int t = 0; t < kTQ; ++t) tmem_st16(lane_base + C::kColQ + 32 * t + 16 * half, qt[t]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_q);
        }
        // online instance: the row's reference maximum (log2 units), the
        // quarter's pair barrier and this half's exchange slot
        float m_ref = -INFINITY;
        const uint32_t bar_pair = kOnline ? smem_u32(&on.bar_pair[quarter]) : 0u;
        float* const x_mine = &on.xchg[quarter][0][half][lane];  // + 64 per block parity
        const int x_other = 32 - 64 * half;                      // the other half's slot
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
                tmem_load_cols(lane_base + C::kColS + kCols * half, r);
#pragma unroll
                for (int i = 0; i < kCols; ++i) s[i] = __uint_as_float(r[i]);
            }
            float mx = 0.0f;
            if constexpr (kOnline) {
                // this half's block maximum over the keys that exist
                if (j == nkb - 1 && last_valid < kBN) {
                    const int valid = last_valid - kCols * half;
#pragma unroll
                    for (int c = 0; c < kCols; ++c)
                        if (c >= valid) s[c] = -INFINITY;
                }
                mx = fmax3(s[0], s[1], s[2]);
#pragma unroll
                for (int c = 3; c + 1 < kCols; c += 2) mx = fmax3(mx, s[c], s[c + 1]);
                mx = fmaxf(mx, s[kCols - 1]);
                x_mine[64 * (j & 1)] = mx;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_pair);
            }
            if (quarter == 0 && half == 0 && j + 1 < nkb &&
                !uwait(bar_kfull((j + 1) % kSK), ((j + 1) / kSK) & 1)) {
                ok = false;
                break;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_c);
            if (!kOnline && j == nkb - 1 && last_valid < kBN) {
                const int valid = last_valid - kCols * half;
#pragma unroll
                for (int c = 0; c < kCols; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            // online: the factor that brings the sums to a moved reference
            // (< 2^-8 when it moved, else exactly 1)
            float alpha = 1.0f;
            if constexpr (kOnline) {
                if (!uwait(bar_pair, j & 1)) {
                    ok = false;
                    break;
                }
                mx = fmaxf(mx, x_mine[64 * (j & 1) + x_other]);
                if (mx > m_ref + kRescaleLog2) {  // always at j == 0 (m_ref = -inf)
                    if (j > 0) alpha = ex2_approx(m_ref - mx);
                    m_ref = mx;
                }
                const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
#pragma unroll
                for (int c = 0; c < kCols / 2; ++c)
                    f2_unpack(f2_add(f2_pack(s[2 * c], s[2 * c + 1]), nm2), s[2 * c], s[2 * c + 1]);
            }
            uint32_t pt[kTP][kCols / 2];
            auto put = [&](int c, float pa, float pb) {
                uint32_t w[kTP];
                split_terms<kTP>(pa, pb, w);
#pragma unroll
                for (int t = 0; t < kTP; ++t) pt[t][c] = w[t];
            };
#pragma unroll
            for (int c = 0; c < kCols / 2; ++c) put(c, ex2_approx(s[2 * c]), ex2_approx(s[2 * c + 1]));  // 2^-inf = 0
            if (j > 0 && !uwait(bar_pfree, (j - 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (C::kFoldOn && j > 0 && j % kFold == 0) {
                // PV_{j-1} closed a run of kFold blocks: fold [O | l] into the
                // sum (the first fold copies); PV_j then starts afresh. The l
                // column (64) is the same for both halves: half 0 folds it.
                const bool first = j == kFold;
#pragma unroll
                for (int piece = 0; piece < 5; ++piece) {
                    if (piece == 4 && half != 0) break;
                    const uint32_t col = piece < 4 ? 32 * half + 8 * piece : kHeadDim;
                    uint32_t ov[8], av[8];
                    tmem_ld8x2(lane_base + C::kColO + col, lane_base + C::kColA + col, ov, av);
                    if (!first) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) + __uint_as_float(av[i]));
                    }
                    tmem_st8(lane_base + C::kColA + col, ov);
                }
            }
#pragma unroll
            for (int t = 0; t < kTP; ++t) tmem_store_cols(lane_base + C::kColP + (kBN / 2) * t + (kCols / 2) * half, pt[t]);
            if constexpr (kOnline) {
                // Blocks 0..j-1 are in the current run of [O | l] (unless a
                // fold just closed it: PV_j then starts afresh) and, from the
                // first fold on, in the folded sum: bring both to the new
                // reference before PV_j (released by the next bar_c arrival).
                // This thread's part: dims [32*half, +32) and column 64 + half
                // (l, or a zero column).
                if (__any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
                    for (int which = 0; which < (C::kFoldOn ? 2 : 1); ++which) {
                        if (C::kFoldOn && which == 0 && j % kFold == 0) continue;  // the run was folded away
                        if (which == 1 && j < kFold) continue;                     // nothing folded yet
                        const uint32_t base = lane_base + (which == 0 ? C::kColO : C::kColA);
                        uint32_t o[33];
                        tmem_ld32_1(base + 32u * half, base + kHeadDim + half, o);
#pragma unroll
                        for (int i = 0; i < 33; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32_1(base + 32u * half, base + kHeadDim + half, o);
                    }
                }
            }
        }
        if (ok) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_c);
        }
        if (ok && uwait(bar_o, 0)) {
            tc_fence_after();
            uint32_t o[33];  // this thread's 32 output dims and l (column 64)
            tmem_ld32_1(lane_base + C::kColO + 32 * half, lane_base + C::kColO + kHeadDim, o);
            if (C::kFoldOn && nkb > kFold) {  // plus the folded sum
                uint32_t a[33];
                tmem_ld32_1(lane_base + C::kColA + 32 * half, lane_base + C::kColA + kHeadDim, a);
#pragma unroll
                for (int i = 0; i < 33; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) + __uint_as_float(a[i]));
            }
            const float l = __uint_as_float(o[32]);
            if (row_live) {
                if (!(l > 0.0f && l <= 3.0e38f)) atomicOr(prm.status, kStatusRange);
                const long long orow = map_row(prm.out_map, grow);
                if constexpr (C::kBf16Out) {
                    // bf16 output (round to nearest even) of o / l
                    const float inv = 1.0f / l;
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(prm.out) + (orow * prm.H + h) * kHeadDim +
                                                          32 * half);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float* f = reinterpret_cast<const float*>(&o[8 * i]);
                        dst[i] = make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv), pack_bf16x2(f[2] * inv, f[3] * inv),
                                            pack_bf16x2(f[4] * inv, f[5] * inv), pack_bf16x2(f[6] * inv, f[7] * inv));
                    }
                } else {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(prm.out) + (orow * prm.H + h) * kHeadDim +
                                                            32 * half);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(__fdiv_rn(__uint_as_float(o[4 * i]), l), __fdiv_rn(__uint_as_float(o[4 * i + 1]), l),
                                             __fdiv_rn(__uint_as_float(o[4 * i + 2]), l), __fdiv_rn(__uint_as_float(o[4 * i + 3]), l));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- host

template <int kTQ, int kTP, bool kOnline>
cudaError_t launch_terms(const AttnProblemF32& p, const Params& prm, cudaStream_t stream) {
    constexpr int kBN = Cfg<kTQ, kTP>::kBN;
    const uint64_t nk = static_cast<uint64_t>(p.n_seg) * p.k_len;
    const uint64_t row_bytes = kHeadDim * 2;
    const uint64_t ks = static_cast<uint64_t>(p.k_stride);
    Maps maps{};
    for (int t = 0; t < kTQ; ++t)
        if (!make_map(&maps.k[t], p.k[t], ks, p.H, row_bytes, ks * row_bytes, kBN, 1)) return cudaErrorInvalidValue;
    for (int t = 0; t < kTP; ++t)
        if (!make_map(&maps.v[t], p.v[t], p.H, nk, row_bytes, p.H * row_bytes, 1, kBN)) return cudaErrorInvalidValue;
    // Set once per device (per instance); host threads that race here both set
    // the same attribute, and the flag is published atomically.
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(attn_fwd_f32_kernel<kTQ, kTP, kOnline>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem_bytes<kTQ, kTP, kOnline>()));
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    dim3 grid(p.n_seg * prm.tiles_per_seg, p.H);
    return launch_pdl(attn_fwd_f32_kernel<kTQ, kTP, kOnline>, grid, dim3(kThreads), smem_bytes<kTQ, kTP, kOnline>(), stream,
                      maps, prm);
}

}  // namespace

cudaError_t launch_attention_f32(const AttnProblemF32& p, int* status, long long wait_limit, cudaStream_t stream) {
    const int tp = p.terms_pv == 0 ? p.terms : p.terms_pv;
    if (p.terms != 2 && p.terms != 3) return cudaErrorInvalidValue;
    if (tp != p.terms && !(p.terms == 2 && tp == 1 && p.online)) return cudaErrorInvalidValue;
    if (p.n_seg <= 0 || p.H <= 0 || p.q_len <= 0 || p.k_len <= 0) return cudaSuccess;
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
    prm.out_map = p.out_map;
    if (tp == 1) return launch_terms<2, 1, true>(p, prm, stream);
    if (p.online) return p.terms == 3 ? launch_terms<3, 3, true>(p, prm, stream) : launch_terms<2, 2, true>(p, prm, stream);
    return p.terms == 3 ? launch_terms<3, 3, false>(p, prm, stream) : launch_terms<2, 2, false>(p, prm, stream);
}

}  // namespace vggt
