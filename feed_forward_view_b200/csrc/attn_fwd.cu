// attn_fwd.cu -- FlashAttention-style forward for sm_100a: softmax(Q K^T / 8) V
// over head dim 64, bf16 in / bf16 out, fp32 scores and accumulators.
//
// ("Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V", Section V slides of the
//  VGGT paper-report deck; frame/global key sets from its "Global + Frame
//  Attention" slide; shapes [B, N, 16, 64] from the vggt-jax README table.)
//
// One CTA owns two 128-row query tiles of one head (256 queries) and streams
// that head's keys/values in 96-row blocks:
//
//   warp 0      TMA producer: K_j and V_j together into an 8-slot ring (one
//               full / one empty barrier per slot).
//   warps 1, 2  MMA issuers, one per query tile t. The whole warp runs the
//               loop; one elected lane issues the tcgen05 instructions:
//               S_{t,j} = Q_t K_j^T (TS: Q read from TMEM, M=128 N=96 K=64)
//               and [O_t | l_t] += P_{t,j} [V_j | 1] (TS: P read from TMEM,
//               M=128 N=80 K=96). Both MMAs take their A operand from TMEM,
//               so shared memory only feeds the K and V tiles and every MMA
//               runs at the tensor core's full rate even at these small N.
//   warp 3      idle (completes the first warpgroup).
//   warps 4-11  softmax for tile 0, warps 12-19 for tile 1. A warp may only
//               reach the 32 TMEM lanes of its lane quarter (warp % 4), so each
//               quarter of a tile has two warps that split the key columns:
//               warps 4-7 take score columns 0-47, warps 8-11 columns 48-95
//               (likewise 12-15 / 16-19). Each thread owns one query row (its
//               TMEM lane) and half of its columns: it first copies its half of
//               the row of q_hat from global memory into TMEM; per key block it
//               reads its 48 scores from TMEM, exponentiates them in fp32 and
//               writes P as bf16 to TMEM; finally it normalises its 32 of the
//               64 output dims and stores them. Four softmax warps per scheduler
//               keep the exponential units busier than two, and fill one warp's
//               waits with another's work.
//
// Softmax without a running maximum. softmax is invariant to a common factor
// on every p of a row, so p = 2^(score * log2(e)) with score = q.k / 8 is as
// good as the usual 2^(score * log2(e) - max) as long as nothing overflows or
// underflows. The QK LayerNorm leaves every head vector with Euclidean norm
// below sqrt(64) = 8 (the rotation keeps the norm), so |score| < 8 and
// p lies in [2^-11.6, 2^11.6]: no maximum, no rescaling of O, and the fp32
// sums of up to millions of such terms stay far inside the fp32 range. (The
// kernel reports a row sum that is not a positive finite number in the
// status word, for callers that feed the core other vectors.)
//
// Online softmax (the kOnline instance), for inputs without that bound -- a
// QK LayerNorm with a large learned scale or shift, or any vectors given to
// the core directly. Each row keeps a reference maximum m (log2 units) and
// evaluates p = 2^(score * log2(e) / 8 - m) (FlashAttention's running
// maximum, VGGT slides section V). The reference moves lazily: only when a
// block's maximum exceeds it by more than kRescaleLog2, so that p <= 2^8 in
// between and most blocks need no rescaling at all. When it moves, the
// thread rescales its part of [O | l] in TMEM by 2^(m_old - m_new) after the
// previous PV MMA has finished and before it releases the next one. The two
// softmax warps of a lane quarter hold the two halves of the same rows, and a
// row's two threads must use the same m: per block each writes its half's
// maximum to shared memory and arrives on the quarter's pair barrier, then
// reads the other's after the barrier completes; both then take the same
// decisions from the same values. Q stays unscaled in TMEM (no bf16
// re-rounding of large scores); the scale by log2(e)/8 is part of the
// packed FMA that subtracts m.
//
// Row sums on the tensor core: the PV MMA's B operand is 80 columns wide --
// V_j (64 columns) followed by a constant shared-memory tile whose first
// column is 1 and the rest 0 (the descriptor's leading byte offset points
// from each V slot to it). Column 64 of the accumulator therefore collects
// l = sum_j P_j from the same bf16 P that multiplies V, and the softmax warps
// do no additions of their own.
//
// TMEM columns of tile t (256 each, all 512 used): Q_t [256t, +32) (64 bf16
// per row, two per column), S_t [256t + 32, +96) (fp32), P_t [256t + 128, +48)
// (96 bf16), [O_t | l_t] [256t + 176, +80) (fp32).
//
// One S buffer suffices, and the softmax warps and the issuer meet once per
// block. Right after loading S_{t,j+1} into registers the softmax warps arrive
// on bar_c[t]: P_{t,j} (written at the end of their previous block) is ready
// and S_t is free; the tile's first softmax warp also checks, before it
// arrives, that K_{j+2} has landed. On that signal the issuer issues PV_{t,j}
// and S_{t,j+2} back to back. Both have a whole block of exponentials to
// finish in: PV_{t,j} before P_{t,j+1} overwrites P_t (bar_pfree), S_{t,j+2}
// before the softmax warps come to block j+2 (bar_s). The issuer waits on
// nothing else, because every instruction it executes competes with four busy
// softmax warps for its scheduler: measured, each extra wait there cost
// hundreds of cycles per block even when its barrier had long completed.
//
// The two tiles' issuers take turns (bar_tok): tile 0 issues its group for
// block j after tile 1 issued its group for block j-1, tile 1 after tile 0's
// group j. Left alone, the two tiles drift into step and their groups reach
// the tensor core together, each then waiting behind the other's; taking
// turns offsets the tiles by about one group, so that each group finds the
// tensor core idle and its results come back sooner (measured +4-5%).
//
// bar_c[t] phases: 0 = S_{t,0} read (and K_1 loaded); j + 1 = P_{t,j} written,
// S_{t,j+1} read and K_{j+2} loaded (only P_{t,j} for the last block). Issue
// order for tile t: [Q_t in TMEM, K_0 loaded] S_{t,0}; [bar_c 0] S_{t,1}; then
// for every block j: [bar_c j+1] PV_{t,j}, commit bar_pfree[t] and kv_empty[j's
// slot]; S_{t,j+2}, commit bar_s[t]; at the end, commit bar_o[t]. (K_{j+2}
// reaches the issuer through a chain: the TMA completes its full barrier, the
// checking softmax warp observes it and then releases bar_c, the issuer
// acquires bar_c and only then issues the MMA that reads the tile.)
//
// Barrier phases: a parity wait is unambiguous only while the barrier is at
// most one phase away from the awaited one, in either direction. bar_c,
// bar_s and bar_pfree each complete once per step and the two sides advance
// in lock step: bar_c phase j + 2 needs S_{t,j+2}, which the issuer issues
// only after seeing phase j + 1; bar_s and bar_pfree phases follow issues that
// each need the previous bar_c phase. The K/V ring: slot s is refilled only
// after both tiles committed kv_empty for its previous block.
//
// Every wait is bounded; on timeout the CTA records the timeout in the device
// status word, stops issuing work, drains what it has in flight and frees its
// tensor memory before exiting.
#include <atomic>

#include <cuda.h>
#include <cuda_runtime.h>

#include "attn_common.cuh"

namespace vggt {
namespace {

using attn::drain_wait;
using attn::make_map;
using attn::Waiter;

constexpr int kBM = 128;                          // query rows per tile
constexpr int kBN = 96;                           // keys per block
constexpr int kKVTileBytes = kBN * kHeadDim * 2;  // 12 KB
constexpr int kOCols = kHeadDim + 16;             // O (64) and the row-sum block (16)
// Softmax warps per lane quarter of a tile: 2 = each takes half the score
// columns (16 softmax warps), 1 = one warp takes the whole row (8 warps).
#ifndef VGGT_COL_SPLIT
#define VGGT_COL_SPLIT 2
#endif
constexpr int kColSplit = VGGT_COL_SPLIT;
static_assert(kColSplit == 1 || kColSplit == 2, "one or two softmax warps per lane quarter");
constexpr int kWarpsPerTile = 4 * kColSplit;  // softmax warps of one query tile
constexpr int kCols = kBN / kColSplit;        // score columns per softmax thread

// The two CTA shapes. kTiles = 2: two query tiles share every K/V block and
// the tensor core alternates between them; all 512 TMEM columns, an 8-slot
// ring, one CTA per SM. kTiles = 1: one query tile, 256 TMEM columns, a
// 4-slot ring and 384 threads, so that two CTAs share an SM and one's set-up,
// pipeline fill and drain overlap the other's main loop (short key ranges:
// frame attention, small problems).
// Register split: the cap for the CTA's warps at launch; the TMA/MMA
// warpgroup gives registers up, the softmax warpgroups take them:
//   2 tiles, 2 halves: 128 * 56 + 512 * 104 = 60416 <= 640 * 96;
//   2 tiles, 1 half:   128 * 80 + 256 * 208 = 63488 <= 384 * 168;
//   1 tile, 2 halves:  128 * 48 + 256 * 96 = 30720 <= 384 * 80 (two CTAs per SM);
//   1 tile, 1 half:    128 * 48 + 128 * 208 = 32768 <= 256 * 128.
template <int kTiles>
struct Shape {
    static_assert(kTiles == 1 || kTiles == 2, "one or two query tiles per CTA");
    static constexpr int kStages = kTiles == 2 ? 8 : 4;  // K/V ring depth
    static constexpr int kSoftmaxWarps = kWarpsPerTile * kTiles;
    static constexpr int kThreads = 128 + 32 * kSoftmaxWarps;
    static constexpr int kMinBlocks = kTiles == 2 ? 1 : 2;  // resident CTAs per SM
    static constexpr uint32_t kLaunchRegs = kTiles == 2 ? (kColSplit == 2 ? 96 : 168) : (kColSplit == 2 ? 80 : 128);
    static constexpr uint32_t kRegsControl = kTiles == 2 ? (kColSplit == 2 ? 56 : 80) : 48;
    static constexpr uint32_t kRegsSoftmax = kTiles == 2 ? (kColSplit == 2 ? 104 : 208) : (kColSplit == 2 ? 96 : 208);
    static constexpr uint32_t kTmemCols = 256 * kTiles;
    static_assert(128 * kRegsControl + 32 * kSoftmaxWarps * kRegsSoftmax <= kThreads * kLaunchRegs,
                  "register split exceeds the launch allocation");
    static_assert(kThreads * kLaunchRegs * kMinBlocks <= 65536, "registers for the resident CTAs");
};

// TMEM columns of Q_t, S_t, P_t and [O_t | l_t].
__device__ __forceinline__ constexpr uint32_t col_q(int t) { return 256u * t; }
__device__ __forceinline__ constexpr uint32_t col_s(int t) { return 256u * t + 32u; }
__device__ __forceinline__ constexpr uint32_t col_p(int t) { return 256u * t + 128u; }
__device__ __forceinline__ constexpr uint32_t col_o(int t) { return 256u * t + 176u; }
static_assert(32 + kBN <= 128 && 128 + kBN / 2 <= 176 && 176 + kOCols <= 256,
              "TMEM columns of one tile overlap");

static_assert(kBN / 16 == 6 && kHeadDim / 16 == 4,
              "the MMA group helpers issue 6 PV steps and 4 S steps");

constexpr float kScaleLog2 = 0.125f * 1.4426950408889634f;  // log2(e) / sqrt(64)

// Online instance: the reference maximum moves only when a block's maximum
// exceeds it by more than this (log2 units), so every p stays <= 2^8 and the
// fp32 sums of up to 2^21 such terms far from overflow. Exponents on the FMA
// pipe are floored at kFmaFloor (the polynomial's exponent arithmetic holds
// for x >= -125; 2^-120 is nothing beside the row's largest term, >= 1).
constexpr float kRescaleLog2 = 8.0f;
constexpr float kFmaFloor = -120.0f;

// Exponentials per key block: of every 8 consecutive score pairs,
// kExp2OnFma pairs are evaluated on the FMA pipe (polynomial below) and the
// rest with the MUFU ex2 instruction, so that the two units share the work.
#ifndef VGGT_EXP2_ON_FMA_PER8
#define VGGT_EXP2_ON_FMA_PER8 3
#endif
constexpr int kExp2OnFma = VGGT_EXP2_ON_FMA_PER8;

// 2^f ~ c0 + c1 f + ... + cn f^n on [-1/2, 1/2]: minimax in relative error
// (Remez exchange, fit by fit_exp2_poly.py in this directory). Degree 2
// (used): worst relative error of the whole float32 evaluation over [-24, 8]
// 1.7e-3, about the 2^-9 rounding P takes to bf16 anyway, and one packed FMA
// per pair fewer than degree 3 (7.5e-5): measured +2-3% on the attention
// kernel, relative Frobenius error against the oracle 3.86e-3 instead of
// 3.78e-3 at 36 909 tokens.
#ifndef VGGT_EXP2_DEGREE
#define VGGT_EXP2_DEGREE 2
#endif
constexpr int kExp2Degree = VGGT_EXP2_DEGREE;
static_assert(kExp2Degree == 2 || kExp2Degree == 3, "polynomial degree 2 or 3");
__device__ __forceinline__ constexpr float exp2_coef(int i) {
    return kExp2Degree == 3 ? (i == 0 ? 9.999280572e-01f : i == 1 ? 6.932609677e-01f
                                         : i == 2 ? 2.426111251e-01f : 5.517166853e-02f)
                            : (i == 0 ? 1.000443101e+00f : i == 1 ? 7.034479976e-01f : 2.384289354e-01f);
}
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

template <int kStages>
struct SharedStorage {
    uint8_t kv[kStages][2][kKVTileBytes];  // [slot][K, V], 128B-swizzled
    uint8_t ones[kKVTileBytes];            // [1, 0, ..., 0] per key row, 128B-swizzled
    uint64_t bar_kvfull[kStages];
    uint64_t bar_kvempty[kStages];
    uint64_t bar_q[2];      // [tile]: Q_t copied into TMEM
    uint64_t bar_s[2];      // [tile]: S_{t,j} computed
    uint64_t bar_c[2];      // [tile]: P_{t,j-1} written and S_{t,j} read
    uint64_t bar_pfree[2];  // [tile]: PV_{t,j} finished (P_t free, O_t updated)
    uint64_t bar_o[2];      // [tile]: every MMA of the tile finished (once)
    uint64_t bar_tok[2];    // [tile]: the other tile issued its previous MMA group
    uint32_t tmem_base;
    int abort;
};

// Online instance only, placed after SharedStorage: per (tile, lane quarter)
// the pair barrier of its two softmax warps and their block maxima, double
// buffered by block parity ([tile][quarter][parity][half][lane]).
template <int kTiles>
struct OnlineShared {
    uint64_t bar_pair[kTiles][4];
    float xchg[kTiles][4][2][2][32];
};

template <int kTiles, bool kOnline>
constexpr size_t smem_bytes() {
    return sizeof(SharedStorage<Shape<kTiles>::kStages>) + (kOnline ? sizeof(OnlineShared<kTiles>) : 0) +
           1024;  // + alignment slack
}
static_assert(smem_bytes<2, true>() <= 227 * 1024, "shared memory beyond the per-CTA limit");
// two one-tile CTAs per SM: 228 KB per SM, 1 KB of it reserved per CTA
static_assert(2 * (smem_bytes<1, true>() + 1024) <= 228 * 1024, "two one-tile CTAs do not fit an SM");

struct Params {
    const uint16_t* q_hat;  // head-major, head planes q_stride rows apart
    uint16_t* out;          // [n_seg*q_len, H, 64]
    int* status;            // device status word
    long long wait_limit;
    long long q_stride;     // rows per head plane of q_hat
    int q_len, k_len, H;
    int pairs_per_seg;      // CTAs per segment
    RowMap out_map;         // query row r is stored at output row map_row(out_map, r)
};

// TMEM loads and stores of the widths the two column splits use, picked by
// array size.
template <int N>
__device__ __forceinline__ void tmem_load(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 48 || N == 96, "unsupported width");
    if constexpr (N == 48) tmem_ld48(taddr, r);
    if constexpr (N == 96) tmem_ld96(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_store(uint32_t taddr, const uint32_t (&r)[N]) {
    static_assert(N == 16 || N == 24 || N == 32 || N == 48, "unsupported width");
    if constexpr (N == 16) tmem_st16(taddr, r);
    if constexpr (N == 24) tmem_st24(taddr, r);
    if constexpr (N == 32) tmem_st32(taddr, r);
    if constexpr (N == 48) tmem_st48(taddr, r);
}
// O columns [first, first + N - 1) and l (column 64) of [O | l].
template <int N>
__device__ __forceinline__ void tmem_load_o(uint32_t o_base, uint32_t first, uint32_t (&r)[N]) {
    static_assert(N == 33 || N == 80, "unsupported width");
    if constexpr (N == 33) tmem_ld32_1(o_base + first, o_base + kHeadDim, r);
    if constexpr (N == 80) tmem_ld80(o_base, r);
}

// Two bf16 (low half first) times log2(e)/8, rounded back to bf16 (nearest,
// ties to even). Scaling Q once per tile saves a multiply per score pair in
// every key block; the extra rounding (relative 2^-9 per element of Q) moves
// a score by ~0.002 (log2 units) rms, well inside the rounding P already
// takes when it is stored as bf16.
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t w) {
    const float lo = __uint_as_float(w << 16) * kScaleLog2;
    const float hi = __uint_as_float(w & 0xFFFF0000u) * kScaleLog2;
    return pack_bf16x2(lo, hi);
}

// Which score pairs of a row go to which unit: of every 8 consecutive pairs,
// the first kExp2OnFma are evaluated on the FMA pipe, the rest with MUFU.
constexpr int kPairs = kCols / 2;
constexpr int kFmaPairs = kPairs / 8 * kExp2OnFma;
constexpr int kMufuPairs = kPairs - kFmaPairs;
static_assert(kPairs % 8 == 0, "pairs come in groups of 8");
__device__ __forceinline__ constexpr int fma_pair(int k) {
    return 8 * (k / kExp2OnFma) + k % kExp2OnFma;
}
__device__ __forceinline__ constexpr int mufu_pair(int k) {
    return 8 * (k / (8 - kExp2OnFma)) + kExp2OnFma + k % (8 - kExp2OnFma);
}

// p = 2^x for a thread's kCols scores x, packed to bf16 pairs. The scores
// are already in log2 units (Q was scaled by log2(e)/8 when it was copied to
// TMEM): x = q.k * log2(e) / 8.
//
// 2^x on the FMA pipe, x in [-125, 125]: t = x + 1.5 * 2^23 rounds x to the
// nearest integer j and leaves j in the low mantissa bits of t; -j =
// 1.5 * 2^23 - t exactly; f = x - j exactly (|f| <= 1/2); 2^x = p(f) * 2^j,
// with 2^j applied by adding j << 23 to the bit pattern of p(f). Three packed
// adds and FMAs per pair plus one per polynomial degree.
//
// Instruction order. A warp issues in order; MUFU accepts one warp-wide ex2
// every 8 cycles and a packed FMA holds the FMA pipe for 2. Emitting all the
// MUFU work of a row and then all the polynomial work would leave one unit
// idle at a time. Instead the row is software-pipelined: step k issues the
// ex2 pair of MUFU pair k, then stage d of FMA pair k - d for every stage
// d = 6..0 in flight, then packs MUFU pair k - 2 (whose results have landed
// by then). Every step feeds both units, and each value is used a step after
// it was produced, which hides the units' latencies.
__device__ __forceinline__ void exp_pack_row_mixed(const float (&s)[kCols], uint32_t (&pk)[kPairs]) {
    const uint64_t magic2 = f2_pack(kRoundMagic, kRoundMagic);
    constexpr int kStagesFma = 4 + kExp2Degree;  // t, -j, f, the Horner steps, combine + pack
    constexpr int kSteps = (kMufuPairs + 2 > kFmaPairs + kStagesFma - 1)
                               ? kMufuPairs + 2
                               : kFmaPairs + kStagesFma - 1;
    float p[kCols];
    uint64_t tt[kFmaPairs > 0 ? kFmaPairs : 1], ff[kFmaPairs > 0 ? kFmaPairs : 1],
        y[kFmaPairs > 0 ? kFmaPairs : 1];
#pragma unroll
    for (int k = 0; k < kSteps; ++k) {
        if (k < kMufuPairs) {
            const int c = mufu_pair(k);
            p[2 * c] = ex2_approx(s[2 * c]);
            p[2 * c + 1] = ex2_approx(s[2 * c + 1]);
        }
#pragma unroll
        for (int d = kStagesFma - 1; d >= 0; --d) {
            const int i = k - d;
            if (i < 0 || i >= kFmaPairs) continue;
            const int c = fma_pair(i);
            if (d == 0) {
                tt[i] = f2_add(f2_pack(s[2 * c], s[2 * c + 1]), magic2);
            } else if (d == 1) {
                ff[i] = f2_fma(tt[i], f2_pack(-1.0f, -1.0f), magic2);  // -j
            } else if (d == 2) {
                ff[i] = f2_add(f2_pack(s[2 * c], s[2 * c + 1]), ff[i]);  // f
            } else if (d == 3) {  // the first Horner step
                constexpr float a = exp2_coef(kExp2Degree), b = exp2_coef(kExp2Degree - 1);
                y[i] = f2_fma(f2_pack(a, a), ff[i], f2_pack(b, b));
            } else if (d < 3 + kExp2Degree) {
                const float cf = exp2_coef(kExp2Degree - 1 - (d - 3));
                y[i] = f2_fma(y[i], ff[i], f2_pack(cf, cf));
            } else {
                uint32_t q0, q1, t0, t1;
                u2_unpack(y[i], q0, q1);
                u2_unpack(tt[i], t0, t1);
                pk[c] = pack_bf16x2(__uint_as_float(q0 + (t0 << 23)), __uint_as_float(q1 + (t1 << 23)));
            }
        }
        if (k >= 2 && k - 2 < kMufuPairs) {
            const int c = mufu_pair(k - 2);
            pk[c] = pack_bf16x2(p[2 * c], p[2 * c + 1]);
        }
    }
}

// MUFU only: the last block, whose masked scores are -inf (2^-inf = 0).
__device__ __forceinline__ void exp_pack_row_mufu(const float (&s)[kCols], uint32_t (&pk)[kPairs]) {
#pragma unroll
    for (int c = 0; c < kPairs; ++c) pk[c] = pack_bf16x2(ex2_approx(s[2 * c]), ex2_approx(s[2 * c + 1]));
}

// Online instance: the largest of the thread's scores (masked ones -inf).
__device__ __forceinline__ float row_max(const float (&s)[kCols]) {
    float m = fmax3(s[0], s[1], s[2]);
#pragma unroll
    for (int c = 3; c + 1 < kCols; c += 2) m = fmax3(m, s[c], s[c + 1]);
    if constexpr (kCols % 2 == 0) m = fmaxf(m, s[kCols - 1]);
    return m;
}

// Online instance: x = score * log2(e)/8 - m in place, one packed FMA per
// pair; kFloor: the pairs the FMA-pipe polynomial takes are floored at
// kFmaFloor (not for the masked last block, which uses MUFU alone and whose
// -inf must stay -inf).
template <bool kFloor>
__device__ __forceinline__ void shift_scores(float (&s)[kCols], float m) {
    const uint64_t c2 = f2_pack(kScaleLog2, kScaleLog2);
    const uint64_t nm2 = f2_pack(-m, -m);
#pragma unroll
    for (int c = 0; c < kPairs; ++c) f2_unpack(f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), c2, nm2), s[2 * c], s[2 * c + 1]);
    if constexpr (kFloor) {
#pragma unroll
        for (int k = 0; k < kFmaPairs; ++k) {
            const int c = fma_pair(k);
            s[2 * c] = fmaxf(s[2 * c], kFmaFloor);
            s[2 * c + 1] = fmaxf(s[2 * c + 1], kFmaFloor);
        }
    }
}

template <int kTiles, bool kOnline>
__global__ void __launch_bounds__(Shape<kTiles>::kThreads, Shape<kTiles>::kMinBlocks)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const Params prm) {
    griddep_launch_dependents();
    griddep_wait();  // before any global memory access (pdl.cuh)
    using Sh = Shape<kTiles>;
    constexpr int kStages = Sh::kStages;
    constexpr int kThreads = Sh::kThreads;
    extern __shared__ uint8_t smem_raw[];
    SharedStorage<kStages>& sm = *reinterpret_cast<SharedStorage<kStages>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    OnlineShared<kTiles>& on = *reinterpret_cast<OnlineShared<kTiles>*>(&sm + 1);  // online instance only

    // The warp index and the TMEM base go through a lane-0 shuffle so that the
    // compiler knows them to be warp-uniform: everything derived from them
    // (barrier and tile addresses, descriptors) then lives in uniform
    // registers, which tcgen05.mma takes directly. Without that, every MMA
    // first has to move its operands over, which makes each issue several
    // times slower while the softmax warps compete for the same scheduler.
    const int warp = __shfl_sync(0xFFFFFFFFu, static_cast<int>(threadIdx.x >> 5), 0);
    const int lane = threadIdx.x & 31;
    const int seg = blockIdx.x / prm.pairs_per_seg;
    const int pair = blockIdx.x - seg * prm.pairs_per_seg;
    const int h = blockIdx.y;
    const int n_qtiles = (prm.q_len + kBM - 1) / kBM;
    const int tile0 = kTiles * pair;                  // first tile in the segment
    const int ntile = min(kTiles, n_qtiles - tile0);  // 1 or 2
    const int k_row0 = seg * prm.k_len;
    const int nkb = (prm.k_len + kBN - 1) / kBN;
    const int last_valid = prm.k_len - (nkb - 1) * kBN;  // keys in the last block

    // Shared-memory addresses of the barriers and tiles; slot / tile indices
    // are runtime values, so they are formed arithmetically (no local arrays).
    const uint32_t bar_kvfull0 = smem_u32(&sm.bar_kvfull[0]);
    const uint32_t bar_kvempty0 = smem_u32(&sm.bar_kvempty[0]);
    const uint32_t bar_q0 = smem_u32(&sm.bar_q[0]);
    const uint32_t bar_s0 = smem_u32(&sm.bar_s[0]);
    const uint32_t bar_c0 = smem_u32(&sm.bar_c[0]);
    const uint32_t bar_pfree0 = smem_u32(&sm.bar_pfree[0]);
    const uint32_t bar_o0 = smem_u32(&sm.bar_o[0]);
    const uint32_t bar_tok0 = smem_u32(&sm.bar_tok[0]);
    const uint32_t kv_smem0 = smem_u32(sm.kv[0][0]);
    const uint32_t ones_smem = smem_u32(sm.ones);
    auto bar_kvfull = [&](int s) { return bar_kvfull0 + 8u * s; };
    auto bar_kvempty = [&](int s) { return bar_kvempty0 + 8u * s; };
    auto bar_q = [&](int t) { return bar_q0 + 8u * t; };
    auto bar_s = [&](int t) { return bar_s0 + 8u * t; };
    auto bar_c = [&](int t) { return bar_c0 + 8u * t; };
    auto bar_pfree = [&](int t) { return bar_pfree0 + 8u * t; };
    auto bar_o = [&](int t) { return bar_o0 + 8u * t; };
    auto bar_tok = [&](int t) { return bar_tok0 + 8u * t; };
    auto k_smem = [&](int s) { return kv_smem0 + static_cast<uint32_t>(2 * kKVTileBytes) * s; };
    auto v_smem = [&](int s) { return k_smem(s) + static_cast<uint32_t>(kKVTileBytes); };

    // One-tile CTAs (short key ranges, where a CTA's start is a large share of
    // its life) request their first data before the set-up below, so that the
    // loads' latency runs under it: the softmax warps their rows of q_hat
    // (this thread's half of its row: 32 bf16 = 16 words, two head dims per
    // word, low half first), the producer the first K/V block. Measured: the
    // first scores ready ~1 us sooner, +2% on frame attention. Two-tile CTAs
    // load after the set-up (the early producer code made ptxas spill there).
    constexpr bool kEarly = kTiles == 1;
    constexpr int kQWords = 32 / kColSplit;  // this thread's 2-dim words of the row
    uint4 q_raw[kQWords / 4];
    if (kEarly && warp >= 4) {
        const int t = (warp - 4) / (4 * kColSplit);
        const int half = ((warp - 4) >> 2) % kColSplit;
        const int row_in_seg = (tile0 + t) * kBM + (warp & 3) * 32 + lane;
        if (t < ntile && row_in_seg < prm.q_len) {
            const long long grow = static_cast<long long>(seg) * prm.q_len + row_in_seg;
            const uint4* src = reinterpret_cast<const uint4*>(
                prm.q_hat + (static_cast<long long>(h) * prm.q_stride + grow) * kHeadDim + 2 * kQWords * half);
#pragma unroll
            for (int i = 0; i < kQWords / 4; ++i) q_raw[i] = __ldg(src + i);
        }
    }
    attn::fill_ones_tile(sm.ones, kKVTileBytes, kThreads);
    fence_proxy_async_smem();  // make the generic-proxy writes visible to the MMA

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_kvfull(s), 1);
            mbar_init(bar_kvempty(s), ntile);  // one commit per tile issuer
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar_q(t), kWarpsPerTile);  // one arrival per softmax warp of the tile
            mbar_init(bar_s(t), 1);
            mbar_init(bar_c(t), kWarpsPerTile);
            mbar_init(bar_pfree(t), 1);
            mbar_init(bar_o(t), 1);
            mbar_init(bar_tok(t), 1);
        }
        if constexpr (kOnline) {
            for (int t = 0; t < kTiles; ++t)
                for (int qr = 0; qr < 4; ++qr) mbar_init(smem_u32(&on.bar_pair[t][qr]), kColSplit);
        }
        sm.abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
        if constexpr (kEarly) {
            // The first block (its slot is empty; this thread is the TMA
            // producer below, which continues with block 1).
            mbar_arrive_expect_tx(bar_kvfull(0), 2 * kKVTileBytes);
            tma_load_3d(k_smem(0), &tm_k, bar_kvfull(0), 0, k_row0, h);
            tma_load_3d(v_smem(0), &tm_v, bar_kvfull(0), 0, h, k_row0);
        }
    }
    if (!kEarly && warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), Sh::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = __shfl_sync(0xFFFFFFFFu, sm.tmem_base, 0);
    const Waiter wait{prm.wait_limit, &sm.abort, prm.status};

    if (warp < 4) regs_dec<Sh::kRegsControl>();
    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int n_issued = kEarly ? 1 : 0;  // blocks whose loads were started (one-tile: the first at set-up)
            for (int j = n_issued; j < nkb; ++j) {
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
            auto uwait = [&](uint32_t bar, uint32_t parity) {
                return __all_sync(0xFFFFFFFFu, wait(bar, parity)) != 0;
            };
            // S_{t,j} = Q_t K_j^T: 4 steps of 16 head dims; Q_t's 16 dims are
            // 8 TMEM columns, K_j's 32 bytes of each 128-byte row.
            const uint32_t q_tm = tmem + col_q(t);
            const uint32_t s_tm = tmem + col_s(t);
            const uint32_t p_tm = tmem + col_p(t);
            const uint32_t o_tm = tmem + col_o(t);
            auto k_descs = [&](int j, uint64_t (&kd)[4]) {
                const uint64_t base = smem_desc_sw128(k_smem(j % kStages), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) kd[kk] = base + static_cast<uint64_t>((kk * 32) >> 4);
            };
            auto issue_s = [&](const uint64_t (&kd)[4]) {
                if (elect_one()) {
                    tc_fence_after();
                    mma_ts4_commit(s_tm, q_tm, kd, idesc_s, bar_s(t));
                }
                __syncwarp();
            };
            bool ok = uwait(bar_q(t), 0) && uwait(bar_kvfull(0), 0);
            if (ok) {
                uint64_t kd[4];
                k_descs(0, kd);
                issue_s(kd);
            }
            // Phase 0 (S_{t,0} read) is consumed even when there is no S_{t,1}:
            // the loop below waits on phases 1, 2, ... by parity.
            // bar_c phase j also vouches for K_{j+1}: one softmax warp checks
            // that block's full barrier before arriving, so the issuer's one
            // wait per block is this one.
            ok = ok && uwait(bar_c(t), 0);
            if (ok && nkb > 1) {
                uint64_t kd[4];
                k_descs(1, kd);
                issue_s(kd);
            }
            for (int j = 0; ok && j < nkb; ++j) {
                const int s = j % kStages;
                const int jn = j + 2;
                // Every operand of this block's MMAs is ready before the wait,
                // so that once the softmax warps signal, the elected thread
                // only has the MMAs and commits to emit.
                // [O_t | l_t] (+)= P_{t,j} [V_j | 1]: 6 steps of 16 keys. The B
                // operand's second 64-column block (the ones tile) lies a
                // leading byte offset away from the V slot.
                const uint32_t vaddr = v_smem(s);
                const uint64_t vbase = smem_desc_sw128(vaddr, ones_smem - vaddr, 1024);
                uint64_t vd[6];
#pragma unroll
                for (int kk = 0; kk < 6; ++kk) vd[kk] = vbase + static_cast<uint64_t>((kk * 16 * 128) >> 4);
                uint64_t kd[4];
                k_descs(jn, kd);
                const uint32_t pfree = bar_pfree(t);
                const uint32_t empty = bar_kvempty(s);
                if (!uwait(bar_c(t), (j + 1) & 1)) break;
                // The two tiles take turns: tile 0's group j follows tile 1's
                // group j-1, tile 1's group j follows tile 0's group j.
                if (ntile == 2 && (t == 1 || j > 0) &&
                    !uwait(bar_tok(t), (t == 0 ? j - 1 : j) & 1))
                    break;
                if (elect_one()) {
                    tc_fence_after();
                    // P_t free again and O_t includes block j; K_j and V_j no
                    // longer needed by this tile.
                    mma_ts6_commit2(o_tm, p_tm, vd, idesc_o, j > 0 ? 1u : 0u, pfree, empty);
                    if (jn < nkb) mma_ts4_commit(s_tm, q_tm, kd, idesc_s, bar_s(t));
                    if (ntile == 2) mbar_arrive(bar_tok(1 - t));
                }
                __syncwarp();
            }
            // Completes once every MMA of this tile has finished: the softmax
            // warps wait on it before the epilogue; it doubles as the drain.
            if (elect_one()) mma_commit(bar_o(t));
            __syncwarp();
            drain_wait(bar_o(t), 0, prm.wait_limit);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------ softmax
        regs_inc<Sh::kRegsSoftmax>();
        const int t = (warp - 4) / (4 * kColSplit);
        const int half = ((warp - 4) >> 2) % kColSplit;  // score columns [kCols*half, +kCols)
        const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
        const int row = quarter * 32 + lane;
        if (t < ntile) {
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            // Waits are made warp-uniform with a vote: the tcgen05 loads and
            // stores after them need the whole warp.
            auto uwait = [&](uint32_t bar, uint32_t parity) {
                return __all_sync(0xFFFFFFFFu, wait(bar, parity)) != 0;
            };
            const int row_in_seg = (tile0 + t) * kBM + row;
            const bool row_live = row_in_seg < prm.q_len;
            const long long grow = static_cast<long long>(seg) * prm.q_len + row_in_seg;
            // Q_t into TMEM: this thread's half of its row of q_hat (loaded
            // now, or at the start in one-tile CTAs) into its lane, the layout
            // the MMA reads an M x K operand in, each value multiplied by
            // log2(e)/8 on the way (so that S comes out of the MMA in log2
            // units and the exponentials need no multiply). Rows past the
            // segment are zeros and never stored.
            {
                uint32_t qr[kQWords];
                if (row_live) {
                    const uint4* src = reinterpret_cast<const uint4*>(
                        prm.q_hat + (static_cast<long long>(h) * prm.q_stride + grow) * kHeadDim + 2 * kQWords * half);
#pragma unroll
                    for (int i = 0; i < kQWords / 4; ++i) {
                        const uint4 w = kEarly ? q_raw[i] : __ldg(src + i);
                        if constexpr (kOnline) {  // unscaled: the shift applies log2(e)/8 in fp32
                            qr[4 * i] = w.x;
                            qr[4 * i + 1] = w.y;
                            qr[4 * i + 2] = w.z;
                            qr[4 * i + 3] = w.w;
                        } else {
                            qr[4 * i] = scale_bf16x2(w.x);
                            qr[4 * i + 1] = scale_bf16x2(w.y);
                            qr[4 * i + 2] = scale_bf16x2(w.z);
                            qr[4 * i + 3] = scale_bf16x2(w.w);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < kQWords; ++i) qr[i] = 0u;
                }
                tmem_store(lane_base + col_q(t) + kQWords * half, qr);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_q(t));
            }
            // Online instance: the row's reference maximum (log2 units), its
            // pair barrier and the shared-memory slots of its two halves.
            float m_ref = -INFINITY;
            const uint32_t bar_pair = kOnline ? smem_u32(&on.bar_pair[t][quarter]) : 0u;
            float* const x_mine = &on.xchg[t][quarter][0][half][lane];  // + 64 per block parity
            const int x_other = 32 - 64 * half;                         // the other half's slot
            bool ok = true;
            for (int j = 0; j < nkb; ++j) {
                if (!uwait(bar_s(t), j & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float s[kCols];
                {
                    uint32_t r[kCols];
                    tmem_load(lane_base + col_s(t) + kCols * half, r);
#pragma unroll
                    for (int i = 0; i < kCols; ++i) s[i] = __uint_as_float(r[i]);
                }
                const bool masked = j == nkb - 1 && last_valid < kBN;
                float mx = 0.0f;
                if constexpr (kOnline) {
                    // this half's block maximum, over the keys that exist
                    if (masked) {
                        const int valid = last_valid - kCols * half;
#pragma unroll
                        for (int c = 0; c < kCols; ++c)
                            if (c >= valid) s[c] = -INFINITY;
                    }
                    mx = row_max(s);
                    if constexpr (kColSplit == 2) {
                        x_mine[64 * (j & 1)] = mx;
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_pair);
                    }
                }
                // The scores are in registers and P_{t,j-1} is in TMEM: S_t may
                // take S_{t,j+1} and PV_{t,j-1} may run. S_{t,j+1} reads K_{j+1}:
                // the tile's first warp makes sure it has landed before
                // arriving (the ring runs kStages blocks ahead, so this is
                // normally satisfied at once), so that a completed bar_c phase
                // implies it. The issuer, whose every instruction competes with
                // busy softmax warps for its scheduler, then has one barrier
                // per block to wait for.
                if (quarter == 0 && half == 0 && j + 1 < nkb &&
                    !uwait(bar_kvfull((j + 1) % kStages), ((j + 1) / kStages) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_c(t));
                uint32_t pk[kPairs];
                // online: the factor that brings [O | l] to a moved reference
                // (< 2^-8 when it moved, else exactly 1)
                float alpha = 1.0f;
                if constexpr (kOnline) {
                    if constexpr (kColSplit == 2) {
                        // the other half's maximum of the same rows
                        if (!uwait(bar_pair, j & 1)) {
                            ok = false;
                            break;
                        }
                        mx = fmaxf(mx, x_mine[64 * (j & 1) + x_other]);
                    }
                    const float mx2 = mx * kScaleLog2;
                    if (mx2 > m_ref + kRescaleLog2) {  // always at j == 0 (m_ref = -inf)
                        if (j > 0) alpha = ex2_approx(m_ref - mx2);
                        m_ref = mx2;
                    }
                    if (masked)
                        shift_scores<false>(s, m_ref);
                    else
                        shift_scores<true>(s, m_ref);
                }
                if (masked) {
                    if constexpr (!kOnline) {
                        const int valid = last_valid - kCols * half;  // of this thread's columns
#pragma unroll
                        for (int c = 0; c < kCols; ++c)
                            if (c >= valid) s[c] = -INFINITY;
                    }
                    exp_pack_row_mufu(s, pk);
                } else {
                    exp_pack_row_mixed(s, pk);
                }
                // P_t is free once PV_{t,j-1} has finished.
                if (j > 0 && !uwait(bar_pfree(t), (j - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                tmem_store(lane_base + col_p(t) + kPairs * half, pk);
                if constexpr (kOnline) {
                    // [O | l] holds blocks 0..j-1 against the old reference (P is
                    // stored, so its registers are free):
                    // bring this thread's part of it to the new one before
                    // PV_{t,j} adds block j (released by the next bar_c arrival).
                    if (__any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
                        const float a = alpha;
                        if constexpr (kColSplit == 2) {
                            // dims [32*half, +32) and column 64 + half (l, or a zero column)
                            const uint32_t o0 = lane_base + col_o(t) + 32u * half;
                            const uint32_t o1 = lane_base + col_o(t) + kHeadDim + half;
                            uint32_t o[33];
                            tmem_ld32_1(o0, o1, o);
#pragma unroll
                            for (int i = 0; i < 33; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
                            tmem_st32_1(o0, o1, o);
                        } else {
                            uint32_t o[kOCols];
                            tmem_ld80(lane_base + col_o(t), o);
#pragma unroll
                            for (int i = 0; i < kOCols; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
                            tmem_st80(lane_base + col_o(t), o);
                        }
                    }
                }
            }
            if (ok) {
                // P of the last block is in TMEM (there is no next S to read).
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_c(t));
            }
            if (ok && uwait(bar_o(t), 0)) {
                tc_fence_after();
                // This thread's 32 of the 64 output dims, and l (column 64).
                constexpr int kODims = kHeadDim / kColSplit;  // this thread's output dims
                uint32_t o[kColSplit == 2 ? 33 : kOCols];
                tmem_load_o(lane_base + col_o(t), kODims * half, o);
                const float l = __uint_as_float(o[kODims]);
                const float inv = 1.0f / l;
                if (row_live) {
                    // Inputs outside the core's contract can overflow the
                    // max-free softmax; say so instead of storing silently.
                    if (!(l > 0.0f && l <= 3.0e38f)) atomicOr(prm.status, kStatusRange);
                    const long long orow = map_row(prm.out_map, grow);
                    uint4* dst = reinterpret_cast<uint4*>(prm.out + (orow * prm.H + h) * kHeadDim + kODims * half);
#pragma unroll
                    for (int v4 = 0; v4 < kODims / 8; ++v4) {
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
        tmem_dealloc(tmem, Sh::kTmemCols);
    }
}

// ---------------------------------------------------------------- host

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

// Key blocks up to which one query tile per CTA (two CTAs per SM) is used.
// Measured (A/B of the two shapes on the same inputs): one tile wins at 6
// blocks (+21%), 11 (+3.5%) and 15 (+5%: frame attention over 1374-token
// frames), two tiles from 22 blocks on (+7% at 22, +8% at 43, +14% at 115).
#ifndef VGGT_SHORT_KEY_BLOCKS
#define VGGT_SHORT_KEY_BLOCKS 16
#endif
constexpr int kShortKeyBlocks = VGGT_SHORT_KEY_BLOCKS;

template <int kTiles, bool kOnline>
cudaError_t launch_instance(int dev, dim3 grid, const CUtensorMap& tm_k, const CUtensorMap& tm_v, const Params& prm,
                            cudaStream_t stream) {
    using Sh = Shape<kTiles>;
    constexpr size_t smem = smem_bytes<kTiles, kOnline>();
    // Set once per device and instance; host threads that race here both set
    // the same attribute, and the flag is published atomically.
    static std::atomic<bool> attr_set[64];
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        // The register split (setmaxnreg) needs the full launch allocation
        // (kLaunchRegs per thread); with fewer registers the softmax
        // warpgroups' increase could never be granted. Refuse to launch such
        // a build.
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, attn_fwd_kernel<kTiles, kOnline>);
        if (e != cudaSuccess) return e;
        if (static_cast<uint32_t>(fa.numRegs) * Sh::kThreads <
            128 * Sh::kRegsControl + 32 * Sh::kSoftmaxWarps * Sh::kRegsSoftmax)
            return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(attn_fwd_kernel<kTiles, kOnline>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    return launch_pdl(attn_fwd_kernel<kTiles, kOnline>, grid, dim3(Sh::kThreads), smem, stream, tm_k, tm_v, prm);
}

}  // namespace

cudaError_t launch_attention(const AttnProblem& p, int* status, long long wait_limit,
                             cudaStream_t stream) {
    if (p.n_seg <= 0 || p.H <= 0 || p.q_len <= 0 || p.k_len <= 0) return cudaSuccess;
    const uint64_t nk = static_cast<uint64_t>(p.n_seg) * p.k_len;
    const uint64_t row_bytes = kHeadDim * 2;
    const uint64_t ks = static_cast<uint64_t>(p.k_stride);
    CUtensorMap tm_k, tm_v;
    // k_hat: head planes k_stride rows apart -> dims {64, k_stride, H}, box
    // {64, kBN, 1} (rows past a segment's keys are masked in the kernel)
    if (!make_map(&tm_k, p.k_hat, ks, p.H, row_bytes, ks * row_bytes, kBN, 1) ||
        // v: [nk][H][64] -> dims {64, H, nk}, box {64, 1, kBN}
        !make_map(&tm_v, p.v, p.H, nk, row_bytes, p.H * row_bytes, 1, kBN))
        return cudaErrorInvalidValue;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_qtiles = (p.q_len + kBM - 1) / kBM;
    const int nkb = (p.k_len + kBN - 1) / kBN;
    // Two tiles per CTA share every K/V block and keep the tensor core busy
    // while one tile's softmax runs; for short key ranges one tile per CTA,
    // two CTAs per SM, hides each CTA's fixed costs (set-up, the first loads,
    // the drain) behind the other's work, and it doubles the CTA count of
    // grids that would not fill the GPU.
    const long long pair_ctas = static_cast<long long>(p.n_seg) * ((n_qtiles + 1) / 2) * p.H;
    int tiles = (nkb <= kShortKeyBlocks || pair_ctas < sms) ? 1 : 2;
#ifdef VGGT_TILES_PER_CTA
    tiles = VGGT_TILES_PER_CTA;
#endif
    Params prm;
    prm.q_hat = p.q_hat;
    prm.out = p.out;
    prm.status = status;
    prm.wait_limit = wait_limit;
    prm.q_stride = p.q_stride;
    prm.q_len = p.q_len;
    prm.k_len = p.k_len;
    prm.H = p.H;
    prm.out_map = p.out_map;
    prm.pairs_per_seg = (n_qtiles + tiles - 1) / tiles;
    dim3 grid(p.n_seg * prm.pairs_per_seg, p.H);
    if (tiles == 1)
        return p.online ? launch_instance<1, true>(dev, grid, tm_k, tm_v, prm, stream)
                        : launch_instance<1, false>(dev, grid, tm_k, tm_v, prm, stream);
    return p.online ? launch_instance<2, true>(dev, grid, tm_k, tm_v, prm, stream)
                    : launch_instance<2, false>(dev, grid, tm_k, tm_v, prm, stream);
}

cudaError_t launch_wait_probe(int* status, long long wait_limit, cudaStream_t stream) {
    wait_probe_kernel<<<1, 32, 0, stream>>>(status, wait_limit);
    return cudaPeekAtLastError();
}

}  // namespace vggt
