// qk_prologue.cu -- per-head QK LayerNorm (+ optional affine) followed by 2D
// rotary embedding, for one or two token-major tensors per launch; the
// arithmetic is in prologue.cuh.
//
// The result is written head-major [H, n, 64] bf16 (round to nearest even)
// so the attention kernel can fetch contiguous 128-row tiles per head.
//
// Memory-bound: one read and one write of 2 KB per token (H = 16).
// Mapping: one warp per token, 8 lanes per head, grid-stride over the tokens
// of both jobs.
#include <atomic>
#include <cmath>

#include "pdl.cuh"
#include "prologue.cuh"

namespace vggt {
namespace {

constexpr int kWarpsPerBlock = 8;

// kAffA / kAffB: whether job a / b has a LayerNorm affine (separate
// instantiations keep the common no-affine kernel at its register count).
template <bool kAffA, bool kAffB>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
qk_prologue_kernel(const __grid_constant__ PrologueJob a, const __grid_constant__ PrologueJob b, int H,
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
            prologue::process_token<kAffA>(a, aff_a, i, H, lane, my_freq);
        else
            prologue::process_token<kAffB>(b, aff_b, i - a.n, H, lane, my_freq);
    }
    griddep_launch_dependents();
}

// One warp per destination row, 16 bytes per lane per step.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, long long n, int chunks, RowMap m) {
    griddep_wait();  // before any global memory access (pdl.cuh)
    const int lane = threadIdx.x & 31;
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
    for (long long c = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); c < n; c += warps) {
        const uint4* s = src + map_row(m, c) * chunks;
        uint4* d = dst + c * chunks;
        for (int i = lane; i < chunks; i += 32) d[i] = __ldg(s + i);
    }
    griddep_launch_dependents();
}

}  // namespace

cudaError_t launch_gather_rows(const uint16_t* src, uint16_t* dst, long long n, int row_elems,
                               const RowMap& m, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long blocks = (n + 7) / 8;
    if (blocks > static_cast<long long>(sms) * 8) blocks = static_cast<long long>(sms) * 8;
    return launch_pdl(gather_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                      reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst), n, row_elems / 8, m);
}

FreqTable rope_freq_table() {
    FreqTable freq;
    for (int j = 0; j < 16; ++j) freq.f[j] = static_cast<float>(std::pow(100.0, -j / 16.0));
    return freq;
}

cudaError_t launch_qk_prologue(const PrologueJob& a, const PrologueJob& b, int H,
                               cudaStream_t stream) {
    const int total = a.n + b.n;
    if (total <= 0) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    auto kernel = a.ln.on ? (b.ln.on ? qk_prologue_kernel<true, true> : qk_prologue_kernel<true, false>)
                          : (b.ln.on ? qk_prologue_kernel<false, true> : qk_prologue_kernel<false, false>);
    // As many blocks as are resident at once (the warps stride over the
    // tokens): a grid beyond that leaves a second, partial wave that starts
    // only as the first one ends, and that the next launch then waits for.
    static std::atomic<int> per_sm_cache[64][4];
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const int inst = (a.ln.on ? 2 : 0) + (b.ln.on ? 1 : 0);
    int per_sm = per_sm_cache[dev][inst].load(std::memory_order_acquire);
    if (per_sm == 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kWarpsPerBlock * 32, 0);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
        per_sm_cache[dev][inst].store(per_sm, std::memory_order_release);
    }
    int blocks = (total + kWarpsPerBlock - 1) / kWarpsPerBlock;
    blocks = blocks < sms * per_sm ? blocks : sms * per_sm;
    return launch_pdl(kernel, dim3(blocks), dim3(kWarpsPerBlock * 32), 0, stream, a, b, H, rope_freq_table());
}

}  // namespace vggt
