// qk_prologue.cu -- per-head QK LayerNorm followed by 2D rotary embedding.
//
// For every token t and head h of a [n, H, 64] bf16 tensor:
//   y = (x - mean) / sqrt(var + 1e-5)         (64 dims, biased variance)
//   half a in {0: dims 0-31 by pos.row, 1: dims 32-63 by pos.col}:
//     (y[j], y[j+16]) of the half turn by theta_j = p_a * 100^(-j/16):
//     y[j]'    = y[j] cos - y[j+16] sin
//     y[j+16]' = y[j+16] cos + y[j] sin
// and the result is written head-major [H, n, 64] bf16 (round to nearest even)
// so the attention kernel can fetch contiguous 128-row tiles per head.
// (LayerNorm: "Norm: Layer Normalization" slide and layer_norm_eps 1e-05 of
//  the VGGT-Omega config.json field table; RoPE base: rope_base 100.0 in the
//  same table; frequency schedule: "Positional Encoding (4/6)" slide.)
//
// Memory-bound: one read and one write of 2 KB per token (H = 16).
// Mapping: one warp per token. Lane l computes the one (sin, cos) pair of the
// token that belongs to (half l/16, frequency l%16); every lane then owns, for
// 4 heads at a time, 8 dims of one head: dims {4u..4u+3} and {4u+16..4u+19}
// of half a, with a = (l%8)/4, u = l%4 -- so both members of each rotation pair
// stay in the same thread and no data moves between lanes for the rotation.
#include <cmath>

#include <cuda_bf16.h>

#include "vggt_internal.h"

namespace vggt {
namespace {

// 100^(-j/16) for j = 0..15 in fp32, passed by value with every launch.
struct FreqTable {
    float f[16];
};

constexpr int kWarpsPerBlock = 8;
constexpr float kEps = 1e-5f;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}

// Up to 16 heads of one token per pass: the lane's two 8-byte pieces of every
// head group are loaded before any arithmetic, so each warp keeps 2 KB of
// loads in flight.
constexpr int kMaxGroups = 4;

struct TokenLoad {
    uint2 w1[kMaxGroups], w2[kMaxGroups];
};

__device__ __forceinline__ void load_token(const PrologueJob& job, int t, int H, int h0, int lane,
                                           int d1, TokenLoad& ld) {
    const uint16_t* xt = job.x + static_cast<size_t>(t) * H * kHeadDim;
#pragma unroll
    for (int g = 0; g < kMaxGroups; ++g) {
        const int h = h0 + 4 * g + (lane >> 3);
        ld.w1[g] = make_uint2(0, 0);
        ld.w2[g] = make_uint2(0, 0);
        if (h < H) {
            ld.w1[g] = __ldg(reinterpret_cast<const uint2*>(xt + h * kHeadDim + d1));
            ld.w2[g] = __ldg(reinterpret_cast<const uint2*>(xt + h * kHeadDim + d1 + 16));
        }
    }
}

// LayerNorm + rotation of one head group (8 lanes = one head), stored
// head-major. Every lane runs it (the shuffles need the whole warp); lanes
// past the last head (live == false) hold zeros and store nothing.
__device__ __forceinline__ void finish_group(const PrologueJob& job, int t, int h, bool live, int d1,
                                             uint2 w1, uint2 w2, const float (&sv)[4],
                                             const float (&cv)[4]) {
    float x1[4] = {bf16_lo(w1.x), bf16_hi(w1.x), bf16_lo(w1.y), bf16_hi(w1.y)};
    float x2[4] = {bf16_lo(w2.x), bf16_hi(w2.x), bf16_lo(w2.y), bf16_hi(w2.y)};
    float sum = (x1[0] + x1[1]) + (x1[2] + x1[3]) + ((x2[0] + x2[1]) + (x2[2] + x2[3]));
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 4);
    const float mean = sum * (1.0f / kHeadDim);
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x1[i] -= mean;
        x2[i] -= mean;
        sq = fmaf(x1[i], x1[i], sq);
        sq = fmaf(x2[i], x2[i], sq);
    }
    sq += __shfl_xor_sync(0xFFFFFFFFu, sq, 1);
    sq += __shfl_xor_sync(0xFFFFFFFFu, sq, 2);
    sq += __shfl_xor_sync(0xFFFFFFFFu, sq, 4);
    const float rstd = rsqrtf(sq * (1.0f / kHeadDim) + kEps);
    float o1[4], o2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float y1 = x1[i] * rstd, y2 = x2[i] * rstd;
        o1[i] = y1 * cv[i] - y2 * sv[i];
        o2[i] = y2 * cv[i] + y1 * sv[i];
    }
    if (live) {
        uint16_t* dst = job.x_hat + (static_cast<size_t>(h) * job.out_stride + t) * kHeadDim;
        *reinterpret_cast<uint2*>(dst + d1) = make_uint2(pack2(o1[0], o1[1]), pack2(o1[2], o1[3]));
        *reinterpret_cast<uint2*>(dst + d1 + 16) =
            make_uint2(pack2(o2[0], o2[1]), pack2(o2[2], o2[3]));
    }
}

// (sin, cos) of the token's 8 angles this lane needs: lane l computes the
// pair of (half l/16, frequency l%16) and the values are shuffled to the lanes
// that own those dims.
__device__ __forceinline__ void token_angles(const PrologueJob& job, int t, int lane, float my_freq,
                                             float (&sv)[4], float (&cv)[4]) {
    const float2 p = reinterpret_cast<const float2*>(job.pos)[t];
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

__device__ __forceinline__ void process_token(const PrologueJob& job, int t, int H, int lane,
                                              float my_freq) {
    const int sub = lane & 7;
    const int d1 = (sub >> 2) * 32 + 4 * (sub & 3);  // first dim of the x1 group; x2 at d1 + 16
    for (int h0 = 0; h0 < H; h0 += 4 * kMaxGroups) {
        TokenLoad ld;
        load_token(job, t, H, h0, lane, d1, ld);
        float sv[4], cv[4];
        token_angles(job, t, lane, my_freq, sv, cv);
#pragma unroll
        for (int g = 0; g < kMaxGroups; ++g) {
            const int h = h0 + 4 * g + (lane >> 3);
            if (h0 + 4 * g < H)  // warp-uniform
                finish_group(job, t, h, h < H, d1, ld.w1[g], ld.w2[g], sv, cv);
        }
    }
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
qk_prologue_kernel(PrologueJob a, PrologueJob b, int H, FreqTable freq) {
    const int lane = threadIdx.x & 31;
    const int warp = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * kWarpsPerBlock;
    const int total = a.n + b.n;
    // this lane's frequency, picked with constant indices (no local memory)
    float my_freq = freq.f[0];
#pragma unroll
    for (int i = 1; i < 16; ++i)
        if ((lane & 15) == i) my_freq = freq.f[i];
    for (int i = warp; i < total; i += nwarps) {
        if (i < a.n)
            process_token(a, i, H, lane, my_freq);
        else
            process_token(b, i - a.n, H, lane, my_freq);
    }
}

}  // namespace

cudaError_t launch_qk_prologue(const PrologueJob& a, const PrologueJob& b, int H,
                               cudaStream_t stream) {
    const int total = a.n + b.n;
    if (total <= 0) return cudaSuccess;
    FreqTable freq;
    for (int j = 0; j < 16; ++j) freq.f[j] = static_cast<float>(std::pow(100.0, -j / 16.0));
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int blocks = (total + kWarpsPerBlock - 1) / kWarpsPerBlock;
    blocks = blocks < sms * 8 ? blocks : sms * 8;
    qk_prologue_kernel<<<blocks, kWarpsPerBlock * 32, 0, stream>>>(a, b, H, freq);
    return cudaPeekAtLastError();
}

}  // namespace vggt
