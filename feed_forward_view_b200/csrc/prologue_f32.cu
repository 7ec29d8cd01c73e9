// prologue_f32.cu -- the QK prologue and the operand split of the fp32 mode.
//
// The fp32 mode takes fp32 q, k, v and evaluates both attention products on
// the bf16 tensor cores with every fp32 operand x carried as two bf16 terms,
// x_hi = bf16(x) and x_lo = bf16(x - x_hi) (x - x_hi is exact in fp32), which
// represent x to about 2^-17 relative. This file writes those operands:
//   q_hat: LayerNorm (+ affine) + 2D RoPE of q in fp32, stored fp32
//          head-major [H, n, 64] (the attention kernel scales and splits it
//          when it copies it into tensor memory);
//   k_hat: the same prologue, stored split: k_hi and k_lo bf16 head-major;
//   v:     split: v_hi and v_lo bf16 token-major [n, H, 64].
// The prologue arithmetic (prologue.cuh) is the bf16 path's, fed with fp32
// inputs. (LayerNorm: "Norm: Layer Normalization" slide; RoPE base 100 and
// eps 1e-5: the VGGT-Omega config.json table; frequency schedule:
// "Positional Encoding (4/6)" slide.)
//
// Memory-bound; one warp per token as in the bf16 prologue, each lane loading
// its 8 dims of a head as two 16-byte pieces.
#include "prologue.cuh"

namespace vggt {
namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const float ah = __bfloat162float(__float2bfloat16_rn(a));
    const float bh = __bfloat162float(__float2bfloat16_rn(b));
    hi = prologue::pack2(ah, bh);
    lo = prologue::pack2(a - ah, b - bh);
}

template <bool kAffine>
__device__ __forceinline__ void process_token_f32(const PrologueJobF32& job, const float* aff, int t, int H,
                                                  int lane, float my_freq) {
    const int d1 = prologue::lane_dim(lane);
    const float* xt = job.x + static_cast<size_t>(t) * H * kHeadDim;
    float sv[4], cv[4];
    prologue::token_angles(reinterpret_cast<const float2*>(job.pos)[t], lane, my_freq, sv, cv);
    for (int h0 = 0; h0 < H; h0 += 4) {  // a warp covers 4 heads
        const int h = h0 + (lane >> 3);
        const bool live = h < H;
        float x1[4] = {0.f, 0.f, 0.f, 0.f}, x2[4] = {0.f, 0.f, 0.f, 0.f};
        if (live) {
            const float4 a = __ldg(reinterpret_cast<const float4*>(xt + h * kHeadDim + d1));
            const float4 b = __ldg(reinterpret_cast<const float4*>(xt + h * kHeadDim + d1 + 16));
            x1[0] = a.x; x1[1] = a.y; x1[2] = a.z; x1[3] = a.w;
            x2[0] = b.x; x2[1] = b.y; x2[2] = b.z; x2[3] = b.w;
        }
        float o1[4], o2[4];
        prologue::norm_rotate<kAffine>(x1, x2, aff, sv, cv, d1, o1, o2);
        if (!live) continue;
        const size_t row = (static_cast<size_t>(h) * job.out_stride + t) * kHeadDim;
        if (job.split) {
            uint32_t h1[2], l1[2], h2[2], l2[2];
            split2(o1[0], o1[1], h1[0], l1[0]);
            split2(o1[2], o1[3], h1[1], l1[1]);
            split2(o2[0], o2[1], h2[0], l2[0]);
            split2(o2[2], o2[3], h2[1], l2[1]);
            uint16_t* hi = static_cast<uint16_t*>(job.out_hi) + row;
            uint16_t* lo = static_cast<uint16_t*>(job.out_lo) + row;
            *reinterpret_cast<uint2*>(hi + d1) = make_uint2(h1[0], h1[1]);
            *reinterpret_cast<uint2*>(hi + d1 + 16) = make_uint2(h2[0], h2[1]);
            *reinterpret_cast<uint2*>(lo + d1) = make_uint2(l1[0], l1[1]);
            *reinterpret_cast<uint2*>(lo + d1 + 16) = make_uint2(l2[0], l2[1]);
        } else {
            float* o = static_cast<float*>(job.out_hi) + row;
            *reinterpret_cast<float4*>(o + d1) = make_float4(o1[0], o1[1], o1[2], o1[3]);
            *reinterpret_cast<float4*>(o + d1 + 16) = make_float4(o2[0], o2[1], o2[2], o2[3]);
        }
    }
}

template <bool kAffA, bool kAffB>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
qk_prologue_f32_kernel(const __grid_constant__ PrologueJobF32 a, const __grid_constant__ PrologueJobF32 b, int H,
                       FreqTable freq) {
    const int lane = threadIdx.x & 31;
    const int warp = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * kWarpsPerBlock;
    const int total = a.n + b.n;
    const float my_freq = prologue::lane_freq(freq, lane);
    __shared__ __align__(16) prologue::SmemAffine sa, sb;
    const float* aff_a = kAffA ? prologue::stage_affine(a.ln, sa) : nullptr;
    const float* aff_b = kAffB ? prologue::stage_affine(b.ln, sb) : nullptr;
    if (kAffA || kAffB) __syncthreads();
    for (int i = warp; i < total; i += nwarps) {
        if (i < a.n)
            process_token_f32<kAffA>(a, aff_a, i, H, lane, my_freq);
        else
            process_token_f32<kAffB>(b, aff_b, i - a.n, H, lane, my_freq);
    }
}

// hi = bf16(x), lo = bf16(x - hi), 4 values per thread per step.
__global__ void __launch_bounds__(256)
split_bf16_kernel(const float4* __restrict__ x, uint2* __restrict__ hi, uint2* __restrict__ lo, long long n4) {
    for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n4; i += static_cast<long long>(gridDim.x) * 256) {
        const float4 v = __ldg(x + i);
        uint2 h, l;
        split2(v.x, v.y, h.x, l.x);
        split2(v.z, v.w, h.y, l.y);
        hi[i] = h;
        lo[i] = l;
    }
}

int sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

}  // namespace

cudaError_t launch_qk_prologue_f32(const PrologueJobF32& a, const PrologueJobF32& b, int H, cudaStream_t stream) {
    const int total = a.n + b.n;
    if (total <= 0 || H <= 0) return cudaSuccess;
    const int sms = sm_count();
    int blocks = (total + kWarpsPerBlock - 1) / kWarpsPerBlock;
    blocks = blocks < sms * 8 ? blocks : sms * 8;
    auto kernel = a.ln.on ? (b.ln.on ? qk_prologue_f32_kernel<true, true> : qk_prologue_f32_kernel<true, false>)
                          : (b.ln.on ? qk_prologue_f32_kernel<false, true> : qk_prologue_f32_kernel<false, false>);
    kernel<<<blocks, kWarpsPerBlock * 32, 0, stream>>>(a, b, H, rope_freq_table());
    return cudaPeekAtLastError();
}

cudaError_t launch_split_bf16(const float* x, uint16_t* hi, uint16_t* lo, long long n, cudaStream_t stream) {
    const long long n4 = n / 4;  // n is a multiple of 64
    if (n4 <= 0) return cudaSuccess;
    long long blocks = (n4 + 255) / 256;
    const long long cap = static_cast<long long>(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    split_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        reinterpret_cast<const float4*>(x), reinterpret_cast<uint2*>(hi), reinterpret_cast<uint2*>(lo), n4);
    return cudaPeekAtLastError();
}

}  // namespace vggt
