// prologue_f32.cu -- the QK prologue and the operand split of the fp32 mode.
//
// The fp32 mode takes fp32 q, k, v and evaluates both attention products on
// the bf16 tensor cores with every fp32 operand x carried as bf16 terms:
// x_0 = bf16(x), x_1 = bf16(x - x_0), and with three terms x_2 = bf16(x - x_0
// - x_1) (each difference is exact in fp32). Two terms represent x to about
// 2^-17 relative; three carry all 24 significant bits of an fp32 value
// (8 + 8 + 8). This file writes those operands:
//   q_hat: LayerNorm (+ affine) + 2D RoPE of q in fp32, stored fp32
//          head-major [H, n, 64] (the attention kernel scales and splits it
//          when it copies it into tensor memory);
//   k_hat: the same prologue, stored as its bf16 terms, one head-major plane
//          per term;
//   v:     its bf16 terms, one token-major [n, H, 64] array per term.
// The prologue arithmetic (prologue.cuh) is the bf16 path's, fed with fp32
// inputs. (LayerNorm: "Norm: Layer Normalization" slide; RoPE base 100 and
// eps 1e-5: the VGGT-Omega config.json table; frequency schedule:
// "Positional Encoding (4/6)" slide.) The same kernel also takes bf16 inputs:
// bf16 calls whose QK LayerNorm affine enlarges the scores beyond what a bf16
// q_hat / k_hat resolves carry q_hat in fp32 and k_hat as two bf16 terms.
//
// Memory-bound; one warp per token as in the bf16 prologue, each lane loading
// its 8 dims of a head as two 16-byte pieces.
#include "pdl.cuh"
#include "prologue.cuh"

namespace vggt {
namespace {

constexpr int kWarpsPerBlock = 8;

// The bf16 terms of two fp32 values (low half first), kTerms of them: each
// term rounds to nearest, the remainders are exact in fp32.
template <int kTerms>
__device__ __forceinline__ void split_terms(float a, float b, uint32_t (&w)[kTerms]) {
#pragma unroll
    for (int i = 0; i < kTerms; ++i) {
        w[i] = prologue::pack2(a, b);
        if (i + 1 < kTerms) {
            a -= __uint_as_float(w[i] << 16);
            b -= __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
}

template <int kTerms>
__device__ __forceinline__ void store_terms(const PrologueJobF32& job, size_t row, int d1, const float (&o1)[4],
                                            const float (&o2)[4]) {
    uint32_t w[4][kTerms];
    split_terms<kTerms>(o1[0], o1[1], w[0]);
    split_terms<kTerms>(o1[2], o1[3], w[1]);
    split_terms<kTerms>(o2[0], o2[1], w[2]);
    split_terms<kTerms>(o2[2], o2[3], w[3]);
#pragma unroll
    for (int i = 0; i < kTerms; ++i) {
        uint16_t* plane = static_cast<uint16_t*>(job.out[i]) + row;
        *reinterpret_cast<uint2*>(plane + d1) = make_uint2(w[0][i], w[1][i]);
        *reinterpret_cast<uint2*>(plane + d1 + 16) = make_uint2(w[2][i], w[3][i]);
    }
}

template <bool kAffine, bool kBf16In>
__device__ __forceinline__ void process_token_f32(const PrologueJobF32& job, const float* aff, int t, int H,
                                                  int lane, float my_freq) {
    const int d1 = prologue::lane_dim(lane);
    const long long src = map_row(job.in_map, t);
    float sv[4], cv[4];
    prologue::token_angles(reinterpret_cast<const float2*>(job.pos)[src], lane, my_freq, sv, cv);
    for (int h0 = 0; h0 < H; h0 += 4) {  // a warp covers 4 heads
        const int h = h0 + (lane >> 3);
        const bool live = h < H;
        float x1[4] = {0.f, 0.f, 0.f, 0.f}, x2[4] = {0.f, 0.f, 0.f, 0.f};
        if (live) {
            const size_t off = (static_cast<size_t>(src) * H + h) * kHeadDim + d1;
            if constexpr (kBf16In) {
                const uint16_t* xt = static_cast<const uint16_t*>(job.x) + off;
                const uint2 a = __ldg(reinterpret_cast<const uint2*>(xt));
                const uint2 b = __ldg(reinterpret_cast<const uint2*>(xt + 16));
                x1[0] = prologue::bf16_lo(a.x); x1[1] = prologue::bf16_hi(a.x);
                x1[2] = prologue::bf16_lo(a.y); x1[3] = prologue::bf16_hi(a.y);
                x2[0] = prologue::bf16_lo(b.x); x2[1] = prologue::bf16_hi(b.x);
                x2[2] = prologue::bf16_lo(b.y); x2[3] = prologue::bf16_hi(b.y);
            } else {
                const float* xt = static_cast<const float*>(job.x) + off;
                const float4 a = __ldg(reinterpret_cast<const float4*>(xt));
                const float4 b = __ldg(reinterpret_cast<const float4*>(xt + 16));
                x1[0] = a.x; x1[1] = a.y; x1[2] = a.z; x1[3] = a.w;
                x2[0] = b.x; x2[1] = b.y; x2[2] = b.z; x2[3] = b.w;
            }
        }
        float o1[4], o2[4];
        prologue::norm_rotate<kAffine, true>(x1, x2, aff, sv, cv, d1, o1, o2);
        if (!live) continue;
        const size_t row = (static_cast<size_t>(h) * job.out_stride + t) * kHeadDim;
        if (job.terms == 2) {
            store_terms<2>(job, row, d1, o1, o2);
        } else if (job.terms == 3) {
            store_terms<3>(job, row, d1, o1, o2);
        } else {
            float* o = static_cast<float*>(job.out[0]) + row;
            *reinterpret_cast<float4*>(o + d1) = make_float4(o1[0], o1[1], o1[2], o1[3]);
            *reinterpret_cast<float4*>(o + d1 + 16) = make_float4(o2[0], o2[1], o2[2], o2[3]);
        }
    }
}

template <bool kAffA, bool kAffB, bool kBf16In>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
qk_prologue_f32_kernel(const __grid_constant__ PrologueJobF32 a, const __grid_constant__ PrologueJobF32 b, int H,
                       FreqTable freq) {
    griddep_wait();  // before any global memory access (pdl.cuh)
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
            process_token_f32<kAffA, kBf16In>(a, aff_a, i, H, lane, my_freq);
        else
            process_token_f32<kAffB, kBf16In>(b, aff_b, i - a.n, H, lane, my_freq);
    }
    griddep_launch_dependents();
}

// The kTerms bf16 terms of x, 4 values per thread per step.
template <int kTerms>
__global__ void __launch_bounds__(256)
split_bf16_kernel(const float4* __restrict__ x, uint2* __restrict__ t0, uint2* __restrict__ t1,
                  uint2* __restrict__ t2, long long n4) {
    griddep_wait();  // before any global memory access (pdl.cuh)
    for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n4; i += static_cast<long long>(gridDim.x) * 256) {
        const float4 v = __ldg(x + i);
        uint32_t a[kTerms], b[kTerms];
        split_terms<kTerms>(v.x, v.y, a);
        split_terms<kTerms>(v.z, v.w, b);
        t0[i] = make_uint2(a[0], b[0]);
        t1[i] = make_uint2(a[1], b[1]);
        if (kTerms == 3) t2[i] = make_uint2(a[kTerms - 1], b[kTerms - 1]);
    }
    griddep_launch_dependents();
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
    if (b.n > 0 && b.x_bf16 != a.x_bf16) return cudaErrorInvalidValue;
    auto kernel = a.x_bf16
        ? (a.ln.on ? (b.ln.on ? qk_prologue_f32_kernel<true, true, true> : qk_prologue_f32_kernel<true, false, true>)
                   : (b.ln.on ? qk_prologue_f32_kernel<false, true, true> : qk_prologue_f32_kernel<false, false, true>))
        : (a.ln.on ? (b.ln.on ? qk_prologue_f32_kernel<true, true, false> : qk_prologue_f32_kernel<true, false, false>)
                   : (b.ln.on ? qk_prologue_f32_kernel<false, true, false> : qk_prologue_f32_kernel<false, false, false>));
    return launch_pdl(kernel, dim3(blocks), dim3(kWarpsPerBlock * 32), 0, stream, a, b, H, rope_freq_table());
}

cudaError_t launch_split_bf16(const float* x, uint16_t* const (&out)[3], int terms, long long n,
                              cudaStream_t stream) {
    const long long n4 = n / 4;  // n is a multiple of 64
    if (n4 <= 0) return cudaSuccess;
    long long blocks = (n4 + 255) / 256;
    const long long cap = static_cast<long long>(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    auto kernel = terms == 3 ? split_bf16_kernel<3> : split_bf16_kernel<2>;
    return launch_pdl(kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                      reinterpret_cast<const float4*>(x), reinterpret_cast<uint2*>(out[0]),
                      reinterpret_cast<uint2*>(out[1]), reinterpret_cast<uint2*>(out[2]), n4);
}

}  // namespace vggt
