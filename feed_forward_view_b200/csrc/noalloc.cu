// noalloc.cu -- global attention for callers that must not allocate device
// memory once they are running: inference loops that reserve their whole
// memory budget at start-up and forbid allocations afterwards (an allocation
// can stall, fail or fragment the pool mid-stream), and processes where the
// stream-ordered allocator is unavailable or switched off. vggt_attn_global
// takes its scratch (the normalised q and k) with cudaMallocAsync; this entry
// point takes it from a fixed array compiled into the library instead.
//
// The array, g_noalloc_scratch, is a file-scope __device__ buffer of
// VGGT_NOALLOC_SCRATCH_BYTES. Every GPU that loads the library holds it until
// the process exits. Host code cannot pass the array's name to a kernel (on
// the host that name is only a stand-in, not a device address), so the first
// call on each device looks up the real device address with
// cudaGetSymbolAddress while that device is current and caches it.
//
// All calls share the one array: calls whose kernels overlap on the GPU (for
// example on two streams without ordering between them) race on it. Nothing in
// it needs to start at zero: the prologue overwrites every byte the attention
// kernel then reads, and rows past the end are never read from it.
#include <atomic>
#include <cmath>
#include <cstdint>

#include <cuda_runtime.h>

#include "vggt_attn.h"
#include "vggt_internal.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[VGGT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
// Host threads may make their first call on a device at the same time: the
// cached address is published atomically (both would store the same value).
std::atomic<void*> g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device; nullptr if the lookup fails.
void* scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void* addr = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!addr) {
        if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) {
            cudaGetLastError();
            return nullptr;
        }
        g_scratch_addr[dev].store(addr, std::memory_order_release);
    }
    return addr;
}

int square_grid_side(int T) {
    const int p = T - VGGT_N_SPECIAL;
    if (p < 0) return -1;
    int g = static_cast<int>(std::lround(std::sqrt(static_cast<double>(p))));
    while (g * g > p) --g;
    while ((g + 1) * (g + 1) <= p) ++g;
    return g * g == p ? g : -1;
}

bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int vggt_attn_global_noalloc(const vggt_bf16* q, const vggt_bf16* k,
                                        const vggt_bf16* v, const float* pos, vggt_bf16* out,
                                        int S, int T, int H, int D, int kv_down,
                                        cudaStream_t stream) {
    if (S < 0 || T < 0 || H < 0 || D < 0) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    if (square_grid_side(T) < 0) return VGGT_ERR_SHAPE;
    if (kv_down != 0 && kv_down != 1) return VGGT_ERR_SHAPE;
    if (H > 65535) return VGGT_ERR_SHAPE;
    // the token count first, so that the byte count below cannot wrap
    if (static_cast<long long>(S) * T > VGGT_MAX_TOKENS) return VGGT_ERR_SHAPE;
    // normalised q and k, head-major bf16: 2 * N * H * D * 2 bytes
    const unsigned long long n = static_cast<unsigned long long>(S) * static_cast<unsigned>(T);
    const unsigned long long plane = n * static_cast<unsigned>(H) * VGGT_HEAD_DIM * sizeof(uint16_t);
    if (2ull * plane > VGGT_NOALLOC_SCRATCH_BYTES) return VGGT_ERR_SHAPE;
    if (S == 0 || H == 0) return VGGT_OK;
    if (!q || !k || !v || !pos || !out) return VGGT_ERR_NULL;
    if (!is_aligned16(q) || !is_aligned16(k) || !is_aligned16(v) ||
        (reinterpret_cast<uintptr_t>(pos) & 7u) != 0 ||
        !is_aligned16(out))
        return VGGT_ERR_UNSUPPORTED;

    void* scratch = scratch_on_current_device();
    int* status = nullptr;
    long long wait_limit = 0;
    if (!scratch || !vggt::device_status_word(&status, &wait_limit)) return VGGT_ERR_CUDA;

    uint16_t* q_hat = static_cast<uint16_t*>(scratch);
    uint16_t* k_hat = q_hat + plane / sizeof(uint16_t);
    const int N = static_cast<int>(n);
    vggt::PrologueJob jq{q, pos, q_hat, N, N};
    vggt::PrologueJob jk{k, pos, k_hat, N, N};
    if (vggt::launch_qk_prologue(jq, jk, H, stream) != cudaSuccess) return VGGT_ERR_CUDA;
    vggt::AttnProblem p{q_hat, k_hat, v, out, 1, N, N, H, N, N};
    if (vggt::launch_attention(p, status, wait_limit, stream) != cudaSuccess) return VGGT_ERR_CUDA;
    return VGGT_OK;
}
