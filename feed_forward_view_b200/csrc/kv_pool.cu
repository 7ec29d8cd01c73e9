// kv_pool.cu -- per-frame K/V descriptors for compressed-descriptor attention
// (FlashVGGT README: global attention over a compact per-frame descriptor set
// obtained by spatially resampling keys and values; --kv_downfactor 4).
//
// Frame s of T = 5 + g*g tokens becomes Tk = 5 + nc*nc tokens, nc = ceil(g/kd):
//   tokens 0..4 (camera + registers) are copied bit for bit;
//   token 5 + cr*nc + cc is cell (cr, cc): patches rows [cr*kd, min(cr*kd+kd, g))
//   x cols [cc*kd, min(cc*kd+kd, g)). Per channel the members are summed in
//   float32 in row-major order, the sum is divided in float32 (IEEE, round to
//   nearest) by the member count, and the quotient is rounded to bf16 (nearest,
//   ties to even). The position is the same float32 mean of member positions.
// The fixed order and correctly rounded division make the result bit-exact.
//
// Memory-bound: every input byte of K and V is read once, the pooled tokens
// are written once. One 128-thread block per output token; thread i owns the
// 16-byte channel chunks i, i+128, ... of K then of V (1024 channels per token
// for H = 16 -> 128 chunks per tensor), so each member token is read with fully
// coalesced 2 KB row loads.
#include <cuda_bf16.h>

#include "vggt_internal.h"

namespace vggt {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ void add8(float (&acc)[8], const uint4 w) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], __uint_as_float(u[i] << 16));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __uint_as_float(u[i] & 0xFFFF0000u));
    }
}

__device__ __forceinline__ uint32_t round2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}

__global__ void __launch_bounds__(kThreads)
kv_pool_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
               const float* __restrict__ pos, uint16_t* __restrict__ k_out,
               uint16_t* __restrict__ v_out, float* __restrict__ pos_out, int T, int Tk, int g,
               int nc, int kd, int chunks /* 16-byte chunks per token per tensor */) {
    const int i = blockIdx.x;  // output token within the frame
    const int s = blockIdx.y;  // frame
    const size_t src0 = static_cast<size_t>(s) * T;
    const size_t dst = static_cast<size_t>(s) * Tk + i;
    const uint4* k4 = reinterpret_cast<const uint4*>(k);
    const uint4* v4 = reinterpret_cast<const uint4*>(v);
    uint4* ko4 = reinterpret_cast<uint4*>(k_out);
    uint4* vo4 = reinterpret_cast<uint4*>(v_out);

    if (i < kNSpecial) {
        for (int c = threadIdx.x; c < 2 * chunks; c += kThreads) {
            const bool is_k = c < chunks;
            const int cc = is_k ? c : c - chunks;
            const uint4 w = (is_k ? k4 : v4)[(src0 + i) * chunks + cc];
            (is_k ? ko4 : vo4)[dst * chunks + cc] = w;
        }
        if (threadIdx.x == 0) {
            pos_out[2 * dst] = pos[2 * (src0 + i)];
            pos_out[2 * dst + 1] = pos[2 * (src0 + i) + 1];
        }
        return;
    }
    const int cell = i - kNSpecial;
    const int cr = cell / nc, cc0 = cell % nc;
    const int r0 = cr * kd, r1 = min(r0 + kd, g);
    const int c0 = cc0 * kd, c1 = min(c0 + kd, g);
    const float count = static_cast<float>((r1 - r0) * (c1 - c0));

    for (int c = threadIdx.x; c < 2 * chunks; c += kThreads) {
        const bool is_k = c < chunks;
        const int ch = is_k ? c : c - chunks;
        const uint4* src = is_k ? k4 : v4;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int r = r0; r < r1; ++r) {
            const size_t row = src0 + kNSpecial + static_cast<size_t>(r) * g;
#pragma unroll 4
            for (int col = c0; col < c1; ++col) add8(acc, src[(row + col) * chunks + ch]);
        }
        uint4 o;
        o.x = round2(__fdiv_rn(acc[0], count), __fdiv_rn(acc[1], count));
        o.y = round2(__fdiv_rn(acc[2], count), __fdiv_rn(acc[3], count));
        o.z = round2(__fdiv_rn(acc[4], count), __fdiv_rn(acc[5], count));
        o.w = round2(__fdiv_rn(acc[6], count), __fdiv_rn(acc[7], count));
        (is_k ? ko4 : vo4)[dst * chunks + ch] = o;
    }
    if (threadIdx.x == 0) {
        float pr = 0.f, pc = 0.f;
        for (int r = r0; r < r1; ++r)
            for (int col = c0; col < c1; ++col) {
                const size_t t = src0 + kNSpecial + static_cast<size_t>(r) * g + col;
                pr = __fadd_rn(pr, pos[2 * t]);
                pc = __fadd_rn(pc, pos[2 * t + 1]);
            }
        pos_out[2 * dst] = __fdiv_rn(pr, count);
        pos_out[2 * dst + 1] = __fdiv_rn(pc, count);
    }
}

}  // namespace

cudaError_t launch_kv_pool(const uint16_t* k, const uint16_t* v, const float* pos,
                           uint16_t* k_out, uint16_t* v_out, float* pos_out, int S, int T,
                           int g, int kd, int H, cudaStream_t stream) {
    const int nc = g > 0 ? (g + kd - 1) / kd : 0;
    const int Tk = kNSpecial + nc * nc;
    if (S <= 0 || H <= 0) return cudaSuccess;
    const int chunks = H * kHeadDim / 8;
    dim3 grid(Tk, S);
    kv_pool_kernel<<<grid, kThreads, 0, stream>>>(k, v, pos, k_out, v_out, pos_out, T, Tk, g, nc,
                                                  kd, chunks);
    return cudaPeekAtLastError();
}

}  // namespace vggt
