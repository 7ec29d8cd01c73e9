// abi.cu -- the extern "C" entry points declared in include/vggt_attn.h.
//
// Each call validates every argument on the host (nothing is launched for an
// invalid call), takes its scratch from the library's stream-ordered memory
// pool on the caller's stream, launches the kernels in stream order and frees
// the scratch with cudaFreeAsync on the same stream. No call synchronises the
// stream. The pool keeps freed memory for the next call (the device's default
// pool returns it to the system at every synchronisation, and taking a
// gigabyte back costs milliseconds of host time per call, during which the
// GPU idles); vggt_release_scratch hands it back on request.
#include <cmath>
#include <new>
#include <cstdint>
#include <cstdio>

#include <cuda_runtime.h>

#include "vggt_attn.h"
#include "vggt_internal.h"

namespace {

using vggt::AttnProblem;
using vggt::PrologueJob;

constexpr long long kDefaultWaitLimit = 1LL << 32;  // SM cycles (~2 s at 2 GHz)
constexpr int kMaxDevices = 64;

__device__ int g_device_status;  // kStatusTimeout / kStatusRange bits, 0 when clear

struct DeviceState {
    int* status = nullptr;  // device address of g_device_status
    long long wait_limit = kDefaultWaitLimit;
    cudaMemPool_t pool = nullptr;  // scratch pool, release threshold at its maximum
};
DeviceState g_dev[kMaxDevices];

// State of the current device, with the status word's device address looked
// up once per device (with that device current).
DeviceState* device_state() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    DeviceState& st = g_dev[dev];
    if (!st.status) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        st.status = static_cast<int*>(p);
    }
    if (!st.pool) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        uint64_t keep = UINT64_MAX;
        if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) {
            cudaGetLastError();
            cudaMemPoolDestroy(pool);
            return nullptr;
        }
        st.pool = pool;
    }
    return &st;
}

int grid_side(int T) {
    const int p = T - VGGT_N_SPECIAL;
    if (p < 0) return -1;
    int g = static_cast<int>(std::lround(std::sqrt(static_cast<double>(p))));
    while (g * g > p) --g;
    while ((g + 1) * (g + 1) <= p) ++g;
    return g * g == p ? g : -1;
}

// Every tensor is read or written with 16-byte vector accesses or by TMA,
// which needs 16-byte aligned global addresses.
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// Positions are read as float2 and written as floats: 8 bytes suffice (a
// frame-aligned slice of a positions array is only 8-byte aligned when its
// first token index is odd).
bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

// Shared checks. Returns VGGT_OK to proceed, 1 for an empty problem, or an
// error status.
int check_common(const void* q, const void* k, const void* v, const void* pos, const void* out,
                 int S, int T, int H, int D) {
    if (S < 0 || T < 0 || H < 0 || D < 0) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    if (grid_side(T) < 0) return VGGT_ERR_SHAPE;
    if (static_cast<long long>(S) * T > VGGT_MAX_TOKENS) return VGGT_ERR_SHAPE;
    if (H > 65535) return VGGT_ERR_SHAPE;
    if (S == 0 || H == 0) return 1;
    if (!q || !k || !v || !pos || !out) return VGGT_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned8(pos) || !aligned16(out))
        return VGGT_ERR_UNSUPPORTED;
    return VGGT_OK;
}

size_t head_plane_bytes(long long n_tokens, int H) {
    return static_cast<size_t>(n_tokens) * H * VGGT_HEAD_DIM * sizeof(uint16_t);
}

int to_status(cudaError_t e) { return e == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA; }

// Prologue on (q, pos) and (k, pos_k), then attention; frees the scratch.
int run_attention(const uint16_t* q, const float* pos, const uint16_t* k, const float* pos_k,
                  const uint16_t* v, uint16_t* out, int n_seg, int q_len, int k_len, int H,
                  void* extra_scratch, cudaStream_t stream) {
    DeviceState* st = device_state();
    if (!st) {
        if (extra_scratch) cudaFreeAsync(extra_scratch, stream);
        return VGGT_ERR_CUDA;
    }
    const long long nq = static_cast<long long>(n_seg) * q_len;
    const long long nk = static_cast<long long>(n_seg) * k_len;
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, head_plane_bytes(nq, H) + head_plane_bytes(nk, H), st->pool,
                                stream) != cudaSuccess) {
        cudaGetLastError();
        if (extra_scratch) cudaFreeAsync(extra_scratch, stream);
        return VGGT_ERR_ALLOC;
    }
    uint16_t* q_hat = static_cast<uint16_t*>(scratch);
    uint16_t* k_hat = q_hat + head_plane_bytes(nq, H) / sizeof(uint16_t);
    PrologueJob jq{q, pos, q_hat, static_cast<int>(nq), nq};
    PrologueJob jk{k, pos_k, k_hat, static_cast<int>(nk), nk};
    int rc = to_status(vggt::launch_qk_prologue(jq, jk, H, stream));
    if (rc == VGGT_OK) {
        AttnProblem p{q_hat, k_hat, v, out, n_seg, q_len, k_len, H, nq, nk};
        rc = to_status(vggt::launch_attention(p, st->status, st->wait_limit, stream));
    }
    cudaFreeAsync(scratch, stream);
    if (extra_scratch) cudaFreeAsync(extra_scratch, stream);
    return rc;
}

}  // namespace

namespace vggt {

bool device_status_word(int** status, long long* wait_limit) {
    DeviceState* st = device_state();
    if (!st) return false;
    *status = st->status;
    *wait_limit = st->wait_limit;
    return true;
}

}  // namespace vggt

extern "C" {

int vggt_attn_frame(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                    vggt_bf16* out, int S, int T, int H, int D, int kv_down, cudaStream_t stream) {
    int rc = check_common(q, k, v, pos, out, S, T, H, D);
    if (rc == VGGT_OK && kv_down != 0 && kv_down != 1) rc = VGGT_ERR_SHAPE;
    if (rc != VGGT_OK) return rc == 1 ? VGGT_OK : rc;
    return run_attention(q, pos, k, pos, v, out, S, T, T, H, nullptr, stream);
}

int vggt_attn_global(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                     vggt_bf16* out, int S, int T, int H, int D, int kv_down, cudaStream_t stream) {
    int rc = check_common(q, k, v, pos, out, S, T, H, D);
    if (rc == VGGT_OK && kv_down != 0 && kv_down != 1) rc = VGGT_ERR_SHAPE;
    if (rc != VGGT_OK) return rc == 1 ? VGGT_OK : rc;
    const int n = S * T;
    return run_attention(q, pos, k, pos, v, out, 1, n, n, H, nullptr, stream);
}

int vggt_qk_prologue(const vggt_bf16* x, const float* pos, vggt_bf16* x_hat, int N, int H, int D,
                     cudaStream_t stream) {
    if (N < 0 || H < 0 || D < 0) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    if (N > VGGT_MAX_TOKENS || H > 65535) return VGGT_ERR_SHAPE;
    if (N == 0 || H == 0) return VGGT_OK;
    if (!x || !pos || !x_hat) return VGGT_ERR_NULL;
    if (!aligned16(x) || !aligned8(pos) || !aligned16(x_hat)) return VGGT_ERR_UNSUPPORTED;
    PrologueJob j{x, pos, x_hat, N, N};
    PrologueJob none{nullptr, nullptr, nullptr, 0, 0};
    return to_status(vggt::launch_qk_prologue(j, none, H, stream));
}

int vggt_attn_core(const vggt_bf16* q_hat, const vggt_bf16* k_hat, const vggt_bf16* v,
                   vggt_bf16* out, int n_seg, int q_len, int k_len, int H, int D,
                   cudaStream_t stream) {
    if (n_seg < 0 || q_len < 0 || k_len < 0 || H < 0 || D < 0) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    if (static_cast<long long>(n_seg) * q_len > VGGT_MAX_TOKENS ||
        static_cast<long long>(n_seg) * k_len > VGGT_MAX_TOKENS || H > 65535)
        return VGGT_ERR_SHAPE;
    if (n_seg == 0 || q_len == 0 || k_len == 0 || H == 0) return VGGT_OK;
    if (!q_hat || !k_hat || !v || !out) return VGGT_ERR_NULL;
    if (!aligned16(q_hat) || !aligned16(k_hat) || !aligned16(v) || !aligned16(out))
        return VGGT_ERR_UNSUPPORTED;
    DeviceState* st = device_state();
    if (!st) return VGGT_ERR_CUDA;
    AttnProblem p{q_hat, k_hat, v, out, n_seg, q_len, k_len, H,
                  static_cast<long long>(n_seg) * q_len, static_cast<long long>(n_seg) * k_len};
    return to_status(vggt::launch_attention(p, st->status, st->wait_limit, stream));
}

int vggt_kv_pool_tokens(int T, int kv_down) {
    const int g = grid_side(T);
    if (g < 0 || kv_down < 1) return VGGT_ERR_SHAPE;
    const int nc = g > 0 ? (g + kv_down - 1) / kv_down : 0;
    return VGGT_N_SPECIAL + nc * nc;
}

int vggt_kv_pool(const vggt_bf16* k, const vggt_bf16* v, const float* pos, vggt_bf16* k_out,
                 vggt_bf16* v_out, float* pos_out, int S, int T, int H, int D, int kv_down,
                 cudaStream_t stream) {
    if (S < 0 || T < 0 || H < 0 || D < 0) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    const int g = grid_side(T);
    if (g < 0 || kv_down < 1) return VGGT_ERR_SHAPE;
    if (static_cast<long long>(S) * T > VGGT_MAX_TOKENS || H > 65535) return VGGT_ERR_SHAPE;
    if (S == 0 || H == 0) return VGGT_OK;
    if (!k || !v || !pos || !k_out || !v_out || !pos_out) return VGGT_ERR_NULL;
    if (!aligned16(k) || !aligned16(v) || !aligned8(pos) || !aligned16(k_out) ||
        !aligned16(v_out) || !aligned8(pos_out))
        return VGGT_ERR_UNSUPPORTED;
    return to_status(vggt::launch_kv_pool(k, v, pos, k_out, v_out, pos_out, S, T, g, kv_down, H,
                                          stream));
}

int vggt_attn_descriptor(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                         const float* pos, vggt_bf16* out, int S, int T, int H, int D, int kv_down,
                         cudaStream_t stream) {
    int rc = check_common(q, k, v, pos, out, S, T, H, D);
    if (rc == VGGT_OK && kv_down < 1) rc = VGGT_ERR_SHAPE;
    if (rc != VGGT_OK) return rc == 1 ? VGGT_OK : rc;
    const int g = grid_side(T);
    const int Tk = vggt_kv_pool_tokens(T, kv_down);
    const long long nk = static_cast<long long>(S) * Tk;
    // pooled k, pooled v, pooled positions
    const size_t kv_bytes = head_plane_bytes(nk, H);
    const size_t pos_bytes = static_cast<size_t>(nk) * 2 * sizeof(float);
    DeviceState* st = device_state();
    if (!st) return VGGT_ERR_CUDA;
    void* pooled = nullptr;
    if (cudaMallocFromPoolAsync(&pooled, 2 * kv_bytes + pos_bytes, st->pool, stream) != cudaSuccess) {
        cudaGetLastError();
        return VGGT_ERR_ALLOC;
    }
    uint16_t* kp = static_cast<uint16_t*>(pooled);
    uint16_t* vp = kp + kv_bytes / sizeof(uint16_t);
    float* pp = reinterpret_cast<float*>(vp + kv_bytes / sizeof(uint16_t));
    rc = to_status(vggt::launch_kv_pool(k, v, pos, kp, vp, pp, S, T, g, kv_down, H, stream));
    if (rc != VGGT_OK) {
        cudaFreeAsync(pooled, stream);
        return rc;
    }
    // Every query row attends to all S*Tk descriptors: one segment.
    return run_attention(q, pos, kp, pp, vp, out, 1, S * T, static_cast<int>(nk), H, pooled,
                         stream);
}

// ------------------------------------------------------------- streaming

struct vggt_desc_cache {
    int device;
    int max_frames, T, H, kv_down, g, Tk;
    long long capacity;  // max_frames * Tk descriptor rows
    int frames;          // frames appended so far
    uint16_t* k_hat;     // [H][capacity][64] normalised pooled keys, head-major
    uint16_t* v;         // [capacity][H][64] pooled values, token-major
    float* pos;          // [capacity][2] cell-mean positions
};

int vggt_desc_cache_create(vggt_desc_cache** cache, int max_frames, int T, int H, int D,
                           int kv_down) {
    if (!cache) return VGGT_ERR_NULL;
    *cache = nullptr;
    if (max_frames < 1 || T < 1 || H < 1 || kv_down < 1 || H > 65535) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    const int g = grid_side(T);
    const int Tk = vggt_kv_pool_tokens(T, kv_down);
    if (g < 0 || Tk < 0) return VGGT_ERR_SHAPE;
    const long long capacity = static_cast<long long>(max_frames) * Tk;
    if (capacity > VGGT_MAX_TOKENS) return VGGT_ERR_SHAPE;
    vggt_desc_cache* c = new (std::nothrow) vggt_desc_cache();
    if (!c) return VGGT_ERR_ALLOC;
    if (cudaGetDevice(&c->device) != cudaSuccess) {
        delete c;
        return VGGT_ERR_CUDA;
    }
    c->max_frames = max_frames;
    c->T = T;
    c->H = H;
    c->kv_down = kv_down;
    c->g = g;
    c->Tk = Tk;
    c->capacity = capacity;
    c->frames = 0;
    const size_t plane = head_plane_bytes(capacity, H);
    void* mem = nullptr;
    if (cudaMalloc(&mem, 2 * plane + static_cast<size_t>(capacity) * 2 * sizeof(float)) != cudaSuccess) {
        cudaGetLastError();
        delete c;
        return VGGT_ERR_ALLOC;
    }
    c->k_hat = static_cast<uint16_t*>(mem);
    c->v = c->k_hat + plane / sizeof(uint16_t);
    c->pos = reinterpret_cast<float*>(c->v + plane / sizeof(uint16_t));
    *cache = c;
    return VGGT_OK;
}

int vggt_desc_cache_destroy(vggt_desc_cache* cache) {
    if (!cache) return VGGT_OK;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return VGGT_ERR_CUDA;
    if (cur != cache->device && cudaSetDevice(cache->device) != cudaSuccess) return VGGT_ERR_CUDA;
    const cudaError_t e = cudaFree(cache->k_hat);
    if (cur != cache->device) cudaSetDevice(cur);
    delete cache;
    return e == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA;
}

int vggt_desc_cache_frames(const vggt_desc_cache* cache) {
    return cache ? cache->frames : VGGT_ERR_NULL;
}

int vggt_desc_cache_reset(vggt_desc_cache* cache) {
    if (!cache) return VGGT_ERR_NULL;
    cache->frames = 0;
    return VGGT_OK;
}

int vggt_attn_descriptor_chunk(vggt_desc_cache* cache, const vggt_bf16* q, const vggt_bf16* k,
                               const vggt_bf16* v, const float* pos, vggt_bf16* out, int C,
                               cudaStream_t stream) {
    if (!cache) return VGGT_ERR_NULL;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return VGGT_ERR_CUDA;
    if (cur != cache->device) return VGGT_ERR_UNSUPPORTED;
    if (C < 0) return VGGT_ERR_SHAPE;
    int rc = check_common(q, k, v, pos, out, C, cache->T, cache->H, VGGT_HEAD_DIM);
    if (rc != VGGT_OK) return rc == 1 ? VGGT_OK : rc;
    if (cache->frames + C > cache->max_frames) return VGGT_ERR_SHAPE;
    DeviceState* st = device_state();
    if (!st) return VGGT_ERR_CUDA;
    const int H = cache->H, T = cache->T, Tk = cache->Tk;
    const long long n_q = static_cast<long long>(C) * T;
    const long long row0 = static_cast<long long>(cache->frames) * Tk;  // first new descriptor
    const long long n_new = static_cast<long long>(C) * Tk;
    // Scratch: the chunk's pooled raw keys [C*Tk, H, 64] and q_hat [H, C*T, 64].
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, head_plane_bytes(n_new, H) + head_plane_bytes(n_q, H),
                                st->pool, stream) != cudaSuccess) {
        cudaGetLastError();
        return VGGT_ERR_ALLOC;
    }
    uint16_t* k_raw = static_cast<uint16_t*>(scratch);
    uint16_t* q_hat = k_raw + head_plane_bytes(n_new, H) / sizeof(uint16_t);
    uint16_t* v_new = cache->v + row0 * H * VGGT_HEAD_DIM;
    float* pos_new = cache->pos + row0 * 2;
    // 1. The chunk's descriptors: pooled values and positions straight into
    //    the cache, pooled keys into scratch ...
    rc = to_status(vggt::launch_kv_pool(k, v, pos, k_raw, v_new, pos_new, C, T, cache->g,
                                        cache->kv_down, H, stream));
    // 2. ... then normalised into the cache's key planes (row0 onwards of
    //    each head's plane), together with the chunk's queries.
    if (rc == VGGT_OK) {
        PrologueJob jq{q, pos, q_hat, static_cast<int>(n_q), n_q};
        PrologueJob jk{k_raw, pos_new, cache->k_hat + row0 * VGGT_HEAD_DIM, static_cast<int>(n_new),
                       cache->capacity};
        rc = to_status(vggt::launch_qk_prologue(jq, jk, H, stream));
    }
    // 3. Every query of the chunk attends to every cached descriptor.
    if (rc == VGGT_OK) {
        AttnProblem p{q_hat, cache->k_hat, cache->v, out, 1, static_cast<int>(n_q),
                      static_cast<int>(row0 + n_new), H, n_q, cache->capacity};
        rc = to_status(vggt::launch_attention(p, st->status, st->wait_limit, stream));
    }
    cudaFreeAsync(scratch, stream);
    if (rc == VGGT_OK) cache->frames += C;
    return rc;
}

int vggt_release_scratch(void) {
    DeviceState* st = device_state();
    if (!st) return VGGT_ERR_CUDA;
    if (cudaMemPoolTrimTo(st->pool, 0) != cudaSuccess) {
        cudaGetLastError();
        return VGGT_ERR_CUDA;
    }
    return VGGT_OK;
}

int vggt_get_device_status(cudaStream_t stream) {
    DeviceState* st = device_state();
    if (!st) return VGGT_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return VGGT_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, st->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return VGGT_ERR_CUDA;
    if (h != 0) {
        const int zero = 0;
        if (cudaMemcpy(st->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return VGGT_ERR_CUDA;
        return (h & vggt::kStatusTimeout) ? VGGT_ERR_TIMEOUT : VGGT_ERR_RANGE;
    }
    return VGGT_OK;
}

const char* vggt_status_string(int status) {
    switch (status) {
        case VGGT_OK: return "VGGT_OK";
        case VGGT_ERR_NULL: return "VGGT_ERR_NULL: a required pointer is NULL";
        case VGGT_ERR_UNSUPPORTED:
            return "VGGT_ERR_UNSUPPORTED: head dimension must be 64, pointers aligned (16 bytes; "
                   "positions 8), and the current device the cache's";
        case VGGT_ERR_SHAPE: return "VGGT_ERR_SHAPE: invalid sizes";
        case VGGT_ERR_ALLOC: return "VGGT_ERR_ALLOC: scratch allocation failed";
        case VGGT_ERR_CUDA: return "VGGT_ERR_CUDA: CUDA call or launch failed";
        case VGGT_ERR_TIMEOUT: return "VGGT_ERR_TIMEOUT: a bounded device wait ran out";
        case VGGT_ERR_RANGE:
            return "VGGT_ERR_RANGE: an attention row sum was not a positive finite number "
                   "(q_hat/k_hat outside the core's norm bound)";
        default: return "unknown vggt_status";
    }
}

long long vggt_set_wait_limit(long long cycles) {
    DeviceState* st = device_state();
    if (!st) return -1;
    const long long prev = st->wait_limit;
    st->wait_limit = cycles < 1 ? kDefaultWaitLimit : cycles;
    return prev;
}

int vggt_debug_wait_timeout(cudaStream_t stream) {
    DeviceState* st = device_state();
    if (!st) return VGGT_ERR_CUDA;
    return to_status(vggt::launch_wait_probe(st->status, st->wait_limit, stream));
}

}  // extern "C"
