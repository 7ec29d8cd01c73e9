// prologue.cuh -- the per-head QK LayerNorm + 2D RoPE arithmetic, shared by
// the prologue kernel (qk_prologue.cu) and the fused pooling + key prologue
// kernel (kv_pool.cu) so that both produce the same bits for the same input.
//
// For one head vector x (64 dims) at position (row, col):
//   y = (x - mean) / sqrt(var + 1e-5)          (biased variance, centered)
//   y = y * gamma + beta                       (optional per-dim affine)
//   half a in {0: dims 0-31 by row, 1: dims 32-63 by col}:
//     (y[j], y[j+16]) of the half turn by theta_j = p_a * 100^(-j/16)
// (LayerNorm: "Norm: Layer Normalization" slide of the VGGT paper-report
//  slides and layer_norm_eps 1e-05 of the VGGT-Omega config.json table; RoPE
//  base: rope_base 100.0 in the same table; frequency schedule: "Positional
//  Encoding (4/6)" slide.)
//
// Lane layout: 8 lanes per head. Lane sub = lane % 8 owns dims
// {d1 .. d1+3} and {d1+16 .. d1+19} with d1 = 32*(sub/4) + 4*(sub%4), so both
// members of every rotation pair stay in one thread. A warp covers 4 heads.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"
#include "vggt_internal.h"

namespace vggt {
namespace prologue {

constexpr float kEps = 1e-5f;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}

// First dim of a lane's low group; the high group is at d1 + 16.
__device__ __forceinline__ int lane_dim(int lane) {
    const int sub = lane & 7;
    return (sub >> 2) * 32 + 4 * (sub & 3);
}

// The affine of a job, staged in shared memory by the block (so that no
// registers hold it): gamma then beta, 64 floats each; null when the job has
// none.
struct SmemAffine {
    float v[2 * kHeadDim];
};

// Copies job affine a into s (all threads of the block call it, followed by
// a __syncthreads before use); returns the staged values.
__device__ __forceinline__ const float* stage_affine(const LnAffine& a, SmemAffine& s) {
    for (int i = threadIdx.x; i < 2 * kHeadDim; i += blockDim.x)
        s.v[i] = i < kHeadDim ? a.gamma[i] : a.beta[i - kHeadDim];
    return s.v;
}

// (sin, cos) of the 8 angles a lane needs at position p = (row, col): lane l
// computes the pair of (half l/16, frequency l%16) and the values are
// shuffled to the lanes that own those dims. Every lane of the warp calls it.
__device__ __forceinline__ void token_angles(float2 p, int lane, float my_freq, float (&sv)[4],
                                             float (&cv)[4]) {
    const float my_pos = (lane < 16) ? p.x : p.y;
    float sn, cs;
    sincosf(my_pos * my_freq, &sn, &cs);
    const int sub = lane & 7, a = sub >> 2, u = sub & 3;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int src = a * 16 + 4 * u + i;
        sv[i] = __shfl_sync(0xFFFFFFFFu, sn, src);
        cv[i] = __shfl_sync(0xFFFFFFFFu, cs, src);
    }
}

// The arithmetic below is written with explicitly rounded operations (no
// contraction left to the compiler) and split into the steps of one "unit" --
// the 8 dims d1..d1+3, d1+16..d1+19 an 8-lane thread owns -- so that a thread
// holding two units (norm_rotate2, the 4-lane layout of the fused pooling
// pass) performs exactly the same operations in the same order and produces
// the same bits. A unit is handled as four pairs of adjacent dims, (d1, d1+1),
// (d1+2, d1+3), (d1+16, d1+17), (d1+18, d1+19): the even dims of the pairs in
// one lane, the odd dims in another. kPacked selects packed two-lane fp32
// instructions (add / mul / fma .rn.f32x2: each lane an ordinary round-to-
// nearest operation, two results per instruction) or the same operations one
// by one: identical results. The prologue kernels take the packed form (they
// are partly issue-bound at the power-capped clock, and it halves their
// arithmetic instructions); the fused pooling pass the scalar one (at its
// 64-register cap the register pairs cost it spills and 1.5%).

// A unit's partial sum: ((x0 + x2) + (x16 + x18)) + ((x1 + x3) + (x17 + x19)).
template <bool kPacked>
__device__ __forceinline__ float unit_sum(const float (&x1)[4], const float (&x2)[4]) {
    if constexpr (kPacked) {
        const uint64_t e = f2_add(f2_add(f2_pack(x1[0], x1[1]), f2_pack(x1[2], x1[3])),
                                  f2_add(f2_pack(x2[0], x2[1]), f2_pack(x2[2], x2[3])));
        float lo, hi;
        f2_unpack(e, lo, hi);
        return __fadd_rn(lo, hi);
    } else {
        return __fadd_rn(__fadd_rn(__fadd_rn(x1[0], x1[2]), __fadd_rn(x2[0], x2[2])),
                         __fadd_rn(__fadd_rn(x1[1], x1[3]), __fadd_rn(x2[1], x2[3])));
    }
}

// Centres a unit on the mean (x + (-mean): the same rounding as x - mean) and
// returns its partial sum of squares: (((x0^2 + x2^2) + x16^2) + x18^2) +
// (((x1^2 + x3^2) + x17^2) + x19^2), each step a fused multiply-add.
template <bool kPacked>
__device__ __forceinline__ float unit_center_sq(float (&x1)[4], float (&x2)[4], float mean) {
    if constexpr (!kPacked) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x1[i] = __fadd_rn(x1[i], -mean);
            x2[i] = __fadd_rn(x2[i], -mean);
        }
        float lo = __fmul_rn(x1[0], x1[0]), hi = __fmul_rn(x1[1], x1[1]);
        lo = __fmaf_rn(x1[2], x1[2], lo);
        hi = __fmaf_rn(x1[3], x1[3], hi);
        lo = __fmaf_rn(x2[0], x2[0], lo);
        hi = __fmaf_rn(x2[1], x2[1], hi);
        lo = __fmaf_rn(x2[2], x2[2], lo);
        hi = __fmaf_rn(x2[3], x2[3], hi);
        return __fadd_rn(lo, hi);
    }
    const uint64_t nm = f2_pack(-mean, -mean);
    const uint64_t a = f2_add(f2_pack(x1[0], x1[1]), nm), b = f2_add(f2_pack(x1[2], x1[3]), nm);
    const uint64_t c = f2_add(f2_pack(x2[0], x2[1]), nm), d = f2_add(f2_pack(x2[2], x2[3]), nm);
    f2_unpack(a, x1[0], x1[1]);
    f2_unpack(b, x1[2], x1[3]);
    f2_unpack(c, x2[0], x2[1]);
    f2_unpack(d, x2[2], x2[3]);
    uint64_t q = f2_mul(a, a);
    q = f2_fma(b, b, q);
    q = f2_fma(c, c, q);
    q = f2_fma(d, d, q);
    float lo, hi;
    f2_unpack(q, lo, hi);
    return __fadd_rn(lo, hi);
}

// Scale (+ affine) and rotation of a unit at first dim d1.
template <bool kAffine, bool kPacked>
__device__ __forceinline__ void unit_finish(const float (&x1)[4], const float (&x2)[4], float rstd, const float* aff,
                                            const float (&sv)[4], const float (&cv)[4], int d1, float (&o1)[4],
                                            float (&o2)[4]) {
    if constexpr (!kPacked) {
        float y1[4], y2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            y1[i] = __fmul_rn(x1[i], rstd);
            y2[i] = __fmul_rn(x2[i], rstd);
        }
        if (kAffine) {
            const volatile float* va = aff;  // (see below)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                y1[i] = __fmaf_rn(y1[i], va[d1 + i], va[kHeadDim + d1 + i]);
                y2[i] = __fmaf_rn(y2[i], va[d1 + 16 + i], va[kHeadDim + d1 + 16 + i]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o1[i] = __fmaf_rn(y1[i], cv[i], __fmul_rn(y2[i], -sv[i]));
            o2[i] = __fmaf_rn(y2[i], cv[i], __fmul_rn(y1[i], sv[i]));
        }
        return;
    }
    const uint64_t r2 = f2_pack(rstd, rstd);
    // y1 pairs (j, j+1) for j = d1, d1 + 2; y2 pairs at j + 16
    uint64_t y1[2] = {f2_mul(f2_pack(x1[0], x1[1]), r2), f2_mul(f2_pack(x1[2], x1[3]), r2)};
    uint64_t y2[2] = {f2_mul(f2_pack(x2[0], x2[1]), r2), f2_mul(f2_pack(x2[2], x2[3]), r2)};
    if (kAffine) {
        // volatile: read from shared memory at each use, so the compiler
        // does not hoist the affine values into registers for the whole token
        // loop
        const volatile float* va = aff;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int j = d1 + 2 * k;
            y1[k] = f2_fma(y1[k], f2_pack(va[j], va[j + 1]), f2_pack(va[kHeadDim + j], va[kHeadDim + j + 1]));
            y2[k] = f2_fma(y2[k], f2_pack(va[j + 16], va[j + 17]),
                           f2_pack(va[kHeadDim + j + 16], va[kHeadDim + j + 17]));
        }
    }
    // (y_j, y_{j+16}) -> (y_j cos - y_{j+16} sin, y_{j+16} cos + y_j sin);
    // -(y_{j+16} sin) is formed as y_{j+16} (-sin), the same value
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint64_t c2 = f2_pack(cv[2 * k], cv[2 * k + 1]);
        const uint64_t s2 = f2_pack(sv[2 * k], sv[2 * k + 1]);
        const uint64_t ns2 = f2_pack(-sv[2 * k], -sv[2 * k + 1]);
        f2_unpack(f2_fma(y1[k], c2, f2_mul(y2[k], ns2)), o1[2 * k], o1[2 * k + 1]);
        f2_unpack(f2_fma(y2[k], c2, f2_mul(y1[k], s2)), o2[2 * k], o2[2 * k + 1]);
    }
}

__device__ __forceinline__ float inv_std(float sq) { return rsqrtf(__fmaf_rn(sq, 1.0f / kHeadDim, kEps)); }

// LayerNorm (+ affine) and rotation of one head (8 lanes) whose 8 dims per
// lane are x1 (dims d1..d1+3) and x2 (d1+16..d1+19); the results, in fp32,
// go to o1 and o2. Every lane of the warp runs it (the shuffles need the
// whole warp); lanes that hold no head hold zeros. kAffine: apply the affine
// staged at aff (gamma[64] then beta[64] in shared memory).
template <bool kAffine, bool kPacked>
__device__ __forceinline__ void norm_rotate(float (&x1)[4], float (&x2)[4], const float* aff, const float (&sv)[4],
                                            const float (&cv)[4], int d1, float (&o1)[4], float (&o2)[4]) {
    float sum = unit_sum<kPacked>(x1, x2);
    sum = __fadd_rn(sum, __shfl_xor_sync(0xFFFFFFFFu, sum, 1));
    sum = __fadd_rn(sum, __shfl_xor_sync(0xFFFFFFFFu, sum, 2));
    sum = __fadd_rn(sum, __shfl_xor_sync(0xFFFFFFFFu, sum, 4));
    const float mean = __fmul_rn(sum, 1.0f / kHeadDim);
    float sq = unit_center_sq<kPacked>(x1, x2, mean);
    sq = __fadd_rn(sq, __shfl_xor_sync(0xFFFFFFFFu, sq, 1));
    sq = __fadd_rn(sq, __shfl_xor_sync(0xFFFFFFFFu, sq, 2));
    sq = __fadd_rn(sq, __shfl_xor_sync(0xFFFFFFFFu, sq, 4));
    unit_finish<kAffine, kPacked>(x1, x2, inv_std(sq), aff, sv, cv, d1, o1, o2);
}

// The same for a thread that holds two adjacent units of a head (4 lanes per
// head): unit a at d1 and unit b at d1 + 4, i.e. dims d1..d1+7 and
// d1+16..d1+23 with d1 = 32*(l/2) + 8*(l%2) for lane l % 4. Its sums are the
// 8-lane sums after their first exchange (units 2k and 2k+1), and its two
// exchanges are their second and third: the same operations, the same bits.
template <bool kAffine, bool kPacked>
__device__ __forceinline__ void norm_rotate2(float (&a1)[4], float (&a2)[4], float (&b1)[4], float (&b2)[4],
                                             const float* aff, const float (&sa)[4], const float (&ca)[4],
                                             const float (&sb)[4], const float (&cb)[4], int d1, float (&oa1)[4],
                                             float (&oa2)[4], float (&ob1)[4], float (&ob2)[4]) {
    float sum = __fadd_rn(unit_sum<kPacked>(a1, a2), unit_sum<kPacked>(b1, b2));
    sum = __fadd_rn(sum, __shfl_xor_sync(0xFFFFFFFFu, sum, 1));
    sum = __fadd_rn(sum, __shfl_xor_sync(0xFFFFFFFFu, sum, 2));
    const float mean = __fmul_rn(sum, 1.0f / kHeadDim);
    float sq = __fadd_rn(unit_center_sq<kPacked>(a1, a2, mean), unit_center_sq<kPacked>(b1, b2, mean));
    sq = __fadd_rn(sq, __shfl_xor_sync(0xFFFFFFFFu, sq, 1));
    sq = __fadd_rn(sq, __shfl_xor_sync(0xFFFFFFFFu, sq, 2));
    const float rstd = inv_std(sq);
    unit_finish<kAffine, kPacked>(a1, a2, rstd, aff, sa, ca, d1, oa1, oa2);
    unit_finish<kAffine, kPacked>(b1, b2, rstd, aff, sb, cb, d1 + 4, ob1, ob2);
}

// (sin, cos) of the angles of the two units of a 4-lane thread (see
// norm_rotate2) at position p, computed like token_angles: lane l computes
// the pair of (half l/16, frequency l%16), and the values are shuffled to
// the lanes that own those dims. Every lane of the warp calls it.
__device__ __forceinline__ void token_angles2(float2 p, int lane, float my_freq, float (&sa)[4], float (&ca)[4],
                                              float (&sb)[4], float (&cb)[4]) {
    const float my_pos = (lane < 16) ? p.x : p.y;
    float sn, cs;
    sincosf(my_pos * my_freq, &sn, &cs);
    const int sub = lane & 3;
    const int src = (sub >> 1) * 16 + 8 * (sub & 1);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        sa[i] = __shfl_sync(0xFFFFFFFFu, sn, src + i);
        ca[i] = __shfl_sync(0xFFFFFFFFu, cs, src + i);
        sb[i] = __shfl_sync(0xFFFFFFFFu, sn, src + 4 + i);
        cb[i] = __shfl_sync(0xFFFFFFFFu, cs, src + 4 + i);
    }
}

// norm_rotate, then the bf16 results stored at dst + d1 and dst + d1 + 16
// (dst = the head vector's 64 outputs) by lanes with live == true.
template <bool kAffine>
__device__ __forceinline__ void norm_rotate_store(float (&x1)[4], float (&x2)[4], const float* aff,
                                                  const float (&sv)[4], const float (&cv)[4], bool live,
                                                  uint16_t* dst, int d1) {
    float o1[4], o2[4];
    norm_rotate<kAffine, true>(x1, x2, aff, sv, cv, d1, o1, o2);
    if (live) {
        *reinterpret_cast<uint2*>(dst + d1) = make_uint2(pack2(o1[0], o1[1]), pack2(o1[2], o1[3]));
        *reinterpret_cast<uint2*>(dst + d1 + 16) = make_uint2(pack2(o2[0], o2[1]), pack2(o2[2], o2[3]));
    }
}

// The prologue results o1 (dims d1..d1+3) and o2 (d1+16..d1+19) as two bf16
// terms: y_0 = bf16(y) at hi + d1 (+16), y_1 = bf16(y - y_0) at lo + d1
// (+16); y - y_0 is exact in fp32.
__device__ __forceinline__ void store_two_terms(uint16_t* hi, uint16_t* lo, int d1, const float (&o1)[4],
                                                const float (&o2)[4]) {
    const uint32_t a0 = pack2(o1[0], o1[1]), a1 = pack2(o1[2], o1[3]);
    const uint32_t b0 = pack2(o2[0], o2[1]), b1 = pack2(o2[2], o2[3]);
    *reinterpret_cast<uint2*>(hi + d1) = make_uint2(a0, a1);
    *reinterpret_cast<uint2*>(hi + d1 + 16) = make_uint2(b0, b1);
    *reinterpret_cast<uint2*>(lo + d1) =
        make_uint2(pack2(o1[0] - bf16_lo(a0), o1[1] - bf16_hi(a0)), pack2(o1[2] - bf16_lo(a1), o1[3] - bf16_hi(a1)));
    *reinterpret_cast<uint2*>(lo + d1 + 16) =
        make_uint2(pack2(o2[0] - bf16_lo(b0), o2[1] - bf16_hi(b0)), pack2(o2[2] - bf16_lo(b1), o2[3] - bf16_hi(b1)));
}

// This lane's RoPE frequency 100^(-(lane%16)/16), chosen from the table with
// constant indices (no local memory).
__device__ __forceinline__ float lane_freq(const FreqTable& freq, int lane) {
    float f = freq.f[0];
#pragma unroll
    for (int i = 1; i < 16; ++i)
        if ((lane & 15) == i) f = freq.f[i];
    return f;
}

// Up to 16 heads of one token per pass: the lane's two 8-byte pieces of every
// head group are loaded before any arithmetic, so each warp keeps 2 KB of
// loads in flight.
constexpr int kMaxGroups = 4;

// Token t of job: normalise and rotate all H heads, store head-major. One
// warp per token; every lane of the warp calls it. aff: the job's staged
// affine, or nullptr.
template <bool kAffine>
__device__ __forceinline__ void process_token(const PrologueJob& job, const float* aff, int t, int H,
                                              int lane, float my_freq) {
    const int d1 = lane_dim(lane);
    const long long src = map_row(job.in_map, t);
    const uint16_t* xt = job.x + static_cast<size_t>(src) * H * kHeadDim;
    for (int h0 = 0; h0 < H; h0 += 4 * kMaxGroups) {
        uint2 w1[kMaxGroups], w2[kMaxGroups];
#pragma unroll
        for (int g = 0; g < kMaxGroups; ++g) {
            const int h = h0 + 4 * g + (lane >> 3);
            w1[g] = make_uint2(0, 0);
            w2[g] = make_uint2(0, 0);
            if (h < H) {
                w1[g] = __ldg(reinterpret_cast<const uint2*>(xt + h * kHeadDim + d1));
                w2[g] = __ldg(reinterpret_cast<const uint2*>(xt + h * kHeadDim + d1 + 16));
            }
        }
        float sv[4], cv[4];
        token_angles(reinterpret_cast<const float2*>(job.pos)[src], lane, my_freq, sv, cv);
#pragma unroll
        for (int g = 0; g < kMaxGroups; ++g) {
            const int h = h0 + 4 * g + (lane >> 3);
            if (h0 + 4 * g < H) {  // warp-uniform
                float x1[4] = {bf16_lo(w1[g].x), bf16_hi(w1[g].x), bf16_lo(w1[g].y), bf16_hi(w1[g].y)};
                float x2[4] = {bf16_lo(w2[g].x), bf16_hi(w2[g].x), bf16_lo(w2[g].y), bf16_hi(w2[g].y)};
                uint16_t* dst = job.x_hat + (static_cast<size_t>(h) * job.out_stride + t) * kHeadDim;
                norm_rotate_store<kAffine>(x1, x2, aff, sv, cv, h < H, dst, d1);
            }
        }
    }
}

}  // namespace prologue
}  // namespace vggt
