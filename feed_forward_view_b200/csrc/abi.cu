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
#include <atomic>
#include <cmath>
#include <mutex>
#include <new>
#include <cstdint>
#include <cstdio>
#include <cstdlib>

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
    std::atomic<bool> status_ready{false};  // status word address looked up
    std::atomic<bool> ready{false};         // and the scratch pool created
    int* status = nullptr;                  // device address of g_device_status
    std::atomic<long long> wait_limit{kDefaultWaitLimit};
    cudaMemPool_t pool = nullptr;  // scratch pool, release threshold at its maximum
};
DeviceState g_dev[kMaxDevices];
std::mutex g_init_mutex;  // serialises the one-time set-up of a device's state

// The current device's state with the status word's device address looked
// up (once per device, with that device current). Creates no memory pool:
// calls that allocate nothing (the core, the no-alloc call, the status and
// wait-limit calls) use this alone.
DeviceState* status_state() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    DeviceState& st = g_dev[dev];
    if (st.status_ready.load(std::memory_order_acquire)) return &st;
    // first call on this device (host threads may race to it): set up once
    std::lock_guard<std::mutex> lock(g_init_mutex);
    if (st.status_ready.load(std::memory_order_relaxed)) return &st;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess || !p) {
        cudaGetLastError();
        return nullptr;
    }
    st.status = static_cast<int*>(p);
    st.status_ready.store(true, std::memory_order_release);
    return &st;
}

// Cap on a scratch pool's size from VGGT_SCRATCH_POOL_MAX_BYTES (a positive
// decimal byte count), read when the pool is created; 0 (the driver's
// default, no cap of its own) when unset or not a positive number. A call
// whose scratch does not fit under the cap returns VGGT_ERR_ALLOC and
// launches nothing.
size_t scratch_pool_cap() {
    const char* text = std::getenv("VGGT_SCRATCH_POOL_MAX_BYTES");
    if (!text || !*text) return 0;
    char* end = nullptr;
    const unsigned long long v = std::strtoull(text, &end, 10);
    if (*end != '\0' || text[0] == '-') return 0;
    return static_cast<size_t>(v);
}

// The current device's state with the scratch pool created as well (once per
// device), for the calls that take scratch from it.
DeviceState* device_state() {
    DeviceState* s = status_state();
    if (!s) return nullptr;
    DeviceState& st = *s;
    if (st.ready.load(std::memory_order_acquire)) return &st;
    std::lock_guard<std::mutex> lock(g_init_mutex);
    if (st.ready.load(std::memory_order_relaxed)) return &st;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    props.maxSize = scratch_pool_cap();
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
    st.ready.store(true, std::memory_order_release);
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
    if (S < 0 || T < 1 || H < 0 || D < 0) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    if (static_cast<long long>(S) * T > VGGT_MAX_TOKENS) return VGGT_ERR_SHAPE;
    if (H > 65535) return VGGT_ERR_SHAPE;
    if (S == 0 || H == 0) return 1;
    if (!q || !k || !v || !pos || !out) return VGGT_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned8(pos) || !aligned16(out))
        return VGGT_ERR_UNSUPPORTED;
    return VGGT_OK;
}

// Frame layout of a call: the caller's, checked against T, or VGGT-1B's
// (5 specials + a square grid) when layout is NULL.
int make_layout(const vggt_frame_layout* layout, int T, vggt::FrameLayout* out) {
    if (!layout) {
        const int g = grid_side(T);
        if (g < 0) return VGGT_ERR_SHAPE;
        *out = vggt::FrameLayout{VGGT_N_SPECIAL, g, g, 0};
        return VGGT_OK;
    }
    const vggt_frame_layout& l = *layout;
    if (l.n_front < 0 || l.grid_h < 0 || l.grid_w < 0 || l.n_back < 0) return VGGT_ERR_SHAPE;
    const long long t = static_cast<long long>(l.n_front) + static_cast<long long>(l.grid_h) * l.grid_w +
                        l.n_back;
    if (t != T) return VGGT_ERR_SHAPE;
    *out = vggt::FrameLayout{l.n_front, l.grid_h, l.grid_w, l.n_back};
    return VGGT_OK;
}

// One LayerNorm affine from host arrays (NULL weight = 1, NULL bias = 0);
// *bound receives max|weight| * 8 + ||bias||_2, a bound on the norm of the
// normalised vector (the unscaled LayerNorm output has norm below 8).
bool make_affine(const float* w, const float* b, vggt::LnAffine* a, double* bound) {
    *a = vggt::LnAffine{};
    a->on = (w || b) ? 1 : 0;
    double wmax = w ? 0.0 : 1.0, b2 = 0.0;
    for (int d = 0; d < VGGT_HEAD_DIM; ++d) {
        const float wd = w ? w[d] : 1.0f, bd = b ? b[d] : 0.0f;
        if (!std::isfinite(wd) || !std::isfinite(bd)) return false;
        a->gamma[d] = wd;
        a->beta[d] = bd;
        wmax = std::fmax(wmax, std::fabs(static_cast<double>(wd)));
        b2 += static_cast<double>(bd) * bd;
    }
    *bound = 8.0 * wmax + std::sqrt(b2);
    return true;
}

// The query and key affines of a call, and which attention path runs them.
//
// With Bq = 8 * max|q_weight| + ||q_bias||_2 (a bound on the norm of a
// normalised query, the plain LayerNorm's being below 8) and Bk likewise,
// every score is at most Bq * Bk / 8 in magnitude, and q_hat / k_hat stored
// in bf16 (2^-9 relative rounding per element) move a score by about
// 2^-9 |q_hat| |k_hat| / 8. The plain LayerNorm keeps both small: the bf16
// kernel then evaluates exp(score) with no row maximum (exact up to rounding:
// softmax ignores a common factor) and its outputs stay within the bf16
// path's error. An affine that enlarges Bq * Bk beyond kPreciseRatio times
// the plain 8 * 8 enlarges that error in proportion (measured on N(0, 1)
// inputs: relative Frobenius error 2.9e-3 at weight 1, 4.3e-3 at 1.25, 5e-3
// at 1.41), and the score range without bound. Such calls run in precise
// mode: q_hat in fp32, k_hat as two bf16 terms (16 significant bits), the
// online softmax (running row maximum), on the term-split attention kernel;
// any finite affine is accepted. Only a weight or bias that is not finite is
// refused.
constexpr double kPreciseRatio = 1.21;  // 1.1^2: weights up to 1.1 on both sides, no bias
struct Norms {
    vggt::LnAffine q, k;
    bool online = false;   // running row maximum (set with precise)
    bool precise = false;  // q_hat fp32, k_hat in two bf16 terms
};
int make_norms(const vggt_qk_norm* n, Norms* out) {
    double bq = 8.0, bk = 8.0;
    if (!make_affine(n ? n->q_weight : nullptr, n ? n->q_bias : nullptr, &out->q, &bq) ||
        !make_affine(n ? n->k_weight : nullptr, n ? n->k_bias : nullptr, &out->k, &bk))
        return VGGT_ERR_UNSUPPORTED;
    out->precise = bq * bk > kPreciseRatio * 64.0;
    out->online = out->precise;
    return VGGT_OK;
}

size_t head_plane_bytes(long long n_tokens, int H) {
    return static_cast<size_t>(n_tokens) * H * VGGT_HEAD_DIM * sizeof(uint16_t);
}

int to_status(cudaError_t e) { return e == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA; }

// Precise mode's operands in scratch: q_hat fp32 [H, nq, 64], then the two
// bf16 terms of k_hat, each a head-major plane (k_stride rows per head).
struct PreciseOperands {
    float* q_hat;
    uint16_t* k_hat[2];
};
// Carves them from the start of `scratch` (4 * head_plane_bytes(nq, H) bytes
// for q_hat and the k planes when nk == nq; in general 2 * plane(nq) + 2 *
// plane(nk)); the k planes hold nk rows per head.
PreciseOperands precise_operands(void* scratch, long long nq, int H, long long nk = -1) {
    if (nk < 0) nk = nq;
    PreciseOperands po;
    po.q_hat = static_cast<float*>(scratch);
    po.k_hat[0] = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(scratch) + 2 * head_plane_bytes(nq, H));
    po.k_hat[1] = po.k_hat[0] + head_plane_bytes(nk, H) / sizeof(uint16_t);
    return po;
}
size_t precise_bytes(long long nq, long long nk, int H) { return 2 * head_plane_bytes(nq, H) + 2 * head_plane_bytes(nk, H); }

// Precise-mode prologue: nq query rows (token q_map(r) of q / q_pos) to
// po.q_hat in fp32, nk key rows (token k_map(r) of k / k_pos) as two bf16
// terms into po.k_hat (k_stride rows per head plane); one launch. nq may be 0.
int precise_prologue(const uint16_t* q, const float* q_pos, long long nq, const vggt::RowMap& q_map,
                     const uint16_t* k, const float* k_pos, long long nk, const vggt::RowMap& k_map,
                     const PreciseOperands& po, long long k_stride, const Norms& norms, int H, cudaStream_t stream) {
    vggt::PrologueJobF32 jq{};
    jq.x = q;
    jq.pos = q_pos;
    jq.out[0] = po.q_hat;
    jq.n = static_cast<int>(nq);
    jq.out_stride = nq;
    jq.ln = norms.q;
    jq.terms = 0;
    jq.x_bf16 = true;
    jq.in_map = q_map;
    vggt::PrologueJobF32 jk{};
    jk.x = k;
    jk.pos = k_pos;
    jk.out[0] = po.k_hat[0];
    jk.out[1] = po.k_hat[1];
    jk.n = static_cast<int>(nk);
    jk.out_stride = k_stride;
    jk.ln = norms.k;
    jk.terms = 2;
    jk.x_bf16 = true;
    jk.in_map = k_map;
    if (nq == 0) return to_status(vggt::launch_qk_prologue_f32(jk, vggt::PrologueJobF32{}, H, stream));
    return to_status(vggt::launch_qk_prologue_f32(jq, jk, H, stream));
}

// Precise-mode attention of po's operands (q_stride / k_stride rows per head
// plane) with the bf16 values v [n_seg*k_len, H, 64] into the bf16 out.
int precise_attention(const PreciseOperands& po, long long k_stride, const uint16_t* v, uint16_t* out, int n_seg,
                      int q_len, int k_len, int H, long long q_stride, const vggt::RowMap& out_map,
                      DeviceState* st, cudaStream_t stream) {
    vggt::AttnProblemF32 p{};
    p.q_hat = po.q_hat;
    p.k[0] = po.k_hat[0];
    p.k[1] = po.k_hat[1];
    p.v[0] = v;
    p.terms = 2;
    p.terms_pv = 1;
    p.online = true;
    p.out = out;
    p.n_seg = n_seg;
    p.q_len = q_len;
    p.k_len = k_len;
    p.H = H;
    p.q_stride = q_stride;
    p.k_stride = k_stride;
    p.out_map = out_map;
    return to_status(vggt::launch_attention_f32(p, st->status, st->wait_limit, stream));
}

// Precise-mode descriptors: pools the S frames of k / v / pos into v_out /
// pos_out and writes the normalised pooled keys (fp32 means, no bf16
// rounding) as two bf16 terms head-major into k_hi / k_lo (k_stride rows per
// head plane).
int precise_pool_keys(const uint16_t* k, const uint16_t* v, const float* pos, int S, int T,
                      const vggt::FrameLayout& L, int kd, int H, uint16_t* k_hi, uint16_t* k_lo, long long k_stride,
                      uint16_t* v_out, float* pos_out, const Norms& norms, cudaStream_t stream) {
    vggt::PoolJob job{};
    job.k = k;
    job.v = v;
    job.pos = pos;
    job.k_out = nullptr;
    job.k_hat = k_hi;
    job.k_hat_lo = k_lo;
    job.k_hat_stride = k_stride;
    job.v_out = v_out;
    job.pos_out = pos_out;
    job.S = S;
    job.T = T;
    job.layout = L;
    job.kd = kd;
    job.H = H;
    job.k_ln = norms.k;
    return to_status(vggt::launch_kv_pool(job, stream));
}

// Frame (n_seg = S, q_len = k_len = T) or global (n_seg = 1, q_len = k_len
// = S*T) attention: prologue on q and k (one launch), then attention; the
// scratch q_hat | k_hat is freed on the stream.
int run_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* pos,
                  uint16_t* out, int n_seg, int len, int H, const Norms& norms, cudaStream_t stream) {
    DeviceState* st = device_state();
    if (!st) return VGGT_ERR_CUDA;
    const long long n = static_cast<long long>(n_seg) * len;
    if (norms.precise) {
        // scratch: q_hat fp32 [H, n, 64] | k_hat terms 0 and 1 [H, n, 64]
        void* scratch = nullptr;
        if (cudaMallocFromPoolAsync(&scratch, 4 * head_plane_bytes(n, H), st->pool, stream) != cudaSuccess) {
            cudaGetLastError();
            return VGGT_ERR_ALLOC;
        }
        PreciseOperands po = precise_operands(scratch, n, H);
        int rc = precise_prologue(q, pos, n, vggt::RowMap{}, k, pos, n, vggt::RowMap{}, po, n, norms, H, stream);
        if (rc == VGGT_OK)
            rc = precise_attention(po, n, v, out, n_seg, len, len, H, n, vggt::RowMap{}, st, stream);
        cudaFreeAsync(scratch, stream);
        return rc;
    }
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, 2 * head_plane_bytes(n, H), st->pool, stream) != cudaSuccess) {
        cudaGetLastError();
        return VGGT_ERR_ALLOC;
    }
    uint16_t* q_hat = static_cast<uint16_t*>(scratch);
    uint16_t* k_hat = q_hat + head_plane_bytes(n, H) / sizeof(uint16_t);
    PrologueJob jq{q, pos, q_hat, static_cast<int>(n), n, norms.q};
    PrologueJob jk{k, pos, k_hat, static_cast<int>(n), n, norms.k};
    int rc = to_status(vggt::launch_qk_prologue(jq, jk, H, stream));
    if (rc == VGGT_OK) {
        AttnProblem p{q_hat, k_hat, v, out, n_seg, len, len, H, n, n};
        p.online = norms.online;
        rc = to_status(vggt::launch_attention(p, st->status, st->wait_limit, stream));
    }
    cudaFreeAsync(scratch, stream);
    return rc;
}

// Frame, global and descriptor calls, with or without the _ex options.
enum class Kind { kFrame, kGlobal, kDescriptor };

// plain == true: the original calls, whose frames are VGGT-1B's (T = 5 +
// g*g). The _ex calls take any T for frame and global attention (they do not
// look at the token order) and the caller's layout for the descriptor.
// B scenes of S frames each (B = 1 for the single-scene calls): global and
// descriptor attention stay within a scene.
int attn_call(Kind kind, bool plain, const uint16_t* q, const uint16_t* k, const uint16_t* v,
              const float* pos, uint16_t* out, int B, int S, int T, int H, int D, int kv_down,
              const vggt_frame_layout* layout, const vggt_qk_norm* norm, cudaStream_t stream);

}  // namespace

namespace vggt {

bool device_status_word(int** status, long long* wait_limit) {
    DeviceState* st = status_state();
    if (!st) return false;
    *status = st->status;
    *wait_limit = st->wait_limit;
    return true;
}

}  // namespace vggt

namespace {

// The descriptor paths' two memory passes: the query prologue of (q, q_pos,
// nq tokens) into q_hat (skipped when nq == 0), then the pooling fused with
// the key prologue -- pools the S frames of k/v/pos into v_out / pos_out and
// writes the normalised pooled keys head-major into k_hat (row r of head h at
// k_hat + (h * k_stride + r) * 64).
int pool_and_prologue(const uint16_t* k, const uint16_t* v, const float* pos, int S, int T,
                      const vggt::FrameLayout& L, int kd, int H, uint16_t* k_hat, long long k_stride,
                      uint16_t* v_out, float* pos_out, const uint16_t* q, const float* q_pos,
                      long long nq, uint16_t* q_hat, const Norms& norms, cudaStream_t stream) {
    vggt::PoolJob job{};
    job.k = k;
    job.v = v;
    job.pos = pos;
    job.k_out = nullptr;
    job.k_hat = k_hat;
    job.k_hat_stride = k_stride;
    job.v_out = v_out;
    job.pos_out = pos_out;
    job.S = S;
    job.T = T;
    job.layout = L;
    job.kd = kd;
    job.H = H;
    job.k_ln = norms.k;
    if (nq > 0) {
        PrologueJob jq{q, q_pos, q_hat, static_cast<int>(nq), nq, norms.q};
        PrologueJob none{};
        const int rc = to_status(vggt::launch_qk_prologue(jq, none, H, stream));
        if (rc != VGGT_OK) return rc;
    }
    return to_status(vggt::launch_kv_pool(job, stream));
}

int attn_call(Kind kind, bool plain, const uint16_t* q, const uint16_t* k, const uint16_t* v,
              const float* pos, uint16_t* out, int B, int S, int T, int H, int D, int kv_down,
              const vggt_frame_layout* layout, const vggt_qk_norm* norm, cudaStream_t stream) {
    if (B < 0 || S < 0) return VGGT_ERR_SHAPE;
    if (B > 0 && S > VGGT_MAX_TOKENS / B) return VGGT_ERR_SHAPE;
    int rc = check_common(q, k, v, pos, out, B * S, T, H, D);
    vggt::FrameLayout L{};
    if ((rc == VGGT_OK || rc == 1) && (plain || kind == Kind::kDescriptor)) {
        const int lrc = make_layout(layout, T, &L);
        if (lrc != VGGT_OK) rc = lrc;
    }
    if ((rc == VGGT_OK || rc == 1) && kind != Kind::kDescriptor && kv_down != 0 && kv_down != 1)
        rc = VGGT_ERR_SHAPE;
    if ((rc == VGGT_OK || rc == 1) && kind == Kind::kDescriptor && kv_down < 1) rc = VGGT_ERR_SHAPE;
    Norms norms;
    if (rc == VGGT_OK || rc == 1) {
        const int nrc = make_norms(norm, &norms);
        if (nrc != VGGT_OK) rc = nrc;
    }
    if (rc != VGGT_OK) return rc == 1 ? VGGT_OK : rc;
    if (kind == Kind::kFrame) return run_attention(q, k, v, pos, out, B * S, T, H, norms, stream);
    if (kind == Kind::kGlobal) return run_attention(q, k, v, pos, out, B, S * T, H, norms, stream);

    const int Tk = L.pooled(kv_down);
    const long long nq = static_cast<long long>(B) * S * T;
    const long long nk = static_cast<long long>(B) * S * Tk;
    DeviceState* st = device_state();
    if (!st) return VGGT_ERR_CUDA;
    if (norms.precise) {
        // scratch: q_hat fp32 | k_hat terms [H, nk, 64] x 2 | pooled v
        // [nk, H, 64] | pooled pos [nk, 2]. The keys are pooled as fp32 means
        // and normalised into the two term planes in the same pass.
        const size_t ops = precise_bytes(nq, nk, H), kb = head_plane_bytes(nk, H);
        void* scratch = nullptr;
        if (cudaMallocFromPoolAsync(&scratch, ops + kb + static_cast<size_t>(nk) * 2 * sizeof(float), st->pool,
                                    stream) != cudaSuccess) {
            cudaGetLastError();
            return VGGT_ERR_ALLOC;
        }
        const PreciseOperands po = precise_operands(scratch, nq, H, nk);
        uint16_t* vp = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(scratch) + ops);
        float* pp = reinterpret_cast<float*>(vp + kb / sizeof(uint16_t));
        rc = precise_prologue(q, pos, nq, vggt::RowMap{}, nullptr, nullptr, 0, vggt::RowMap{}, po, nk, norms, H,
                              stream);
        if (rc == VGGT_OK)
            rc = precise_pool_keys(k, v, pos, B * S, T, L, kv_down, H, po.k_hat[0], po.k_hat[1], nk, vp, pp, norms,
                                   stream);
        if (rc == VGGT_OK)
            rc = precise_attention(po, nk, vp, out, B, S * T, S * Tk, H, nq, vggt::RowMap{}, st, stream);
        cudaFreeAsync(scratch, stream);
        return rc;
    }
    // scratch: q_hat [H, nq, 64] | k_hat [H, nk, 64] | pooled v [nk, H, 64] | pooled pos [nk, 2]
    const size_t q_bytes = head_plane_bytes(nq, H), k_bytes = head_plane_bytes(nk, H);
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, q_bytes + 2 * k_bytes + static_cast<size_t>(nk) * 2 * sizeof(float),
                                st->pool, stream) != cudaSuccess) {
        cudaGetLastError();
        return VGGT_ERR_ALLOC;
    }
    uint16_t* q_hat = static_cast<uint16_t*>(scratch);
    uint16_t* k_hat = q_hat + q_bytes / sizeof(uint16_t);
    uint16_t* vp = k_hat + k_bytes / sizeof(uint16_t);
    float* pp = reinterpret_cast<float*>(vp + k_bytes / sizeof(uint16_t));
    rc = pool_and_prologue(k, v, pos, B * S, T, L, kv_down, H, k_hat, nk, vp, pp, q, pos, nq, q_hat, norms,
                           stream);
    if (rc == VGGT_OK) {
        // every query row attends to all S*Tk descriptors: one segment
        // scene b: its S*T query rows attend to its S*Tk descriptors
        AttnProblem p{q_hat, k_hat, vp, out, B, S * T, S * Tk, H, nq, nk};
        p.online = norms.online;
        rc = to_status(vggt::launch_attention(p, st->status, st->wait_limit, stream));
    }
    cudaFreeAsync(scratch, stream);
    return rc;
}

int kv_pool_call(const uint16_t* k, const uint16_t* v, const float* pos, uint16_t* k_out,
                 uint16_t* v_out, float* pos_out, int S, int T, int H, int D, int kv_down,
                 const vggt_frame_layout* layout, cudaStream_t stream) {
    if (S < 0 || T < 1 || H < 0 || D < 0) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    vggt::FrameLayout L{};
    const int lrc = make_layout(layout, T, &L);
    if (lrc != VGGT_OK) return lrc;
    if (kv_down < 1) return VGGT_ERR_SHAPE;
    if (static_cast<long long>(S) * T > VGGT_MAX_TOKENS || H > 65535) return VGGT_ERR_SHAPE;
    if (S == 0 || H == 0) return VGGT_OK;
    if (!k || !v || !pos || !k_out || !v_out || !pos_out) return VGGT_ERR_NULL;
    if (!aligned16(k) || !aligned16(v) || !aligned8(pos) || !aligned16(k_out) || !aligned16(v_out) ||
        !aligned8(pos_out))
        return VGGT_ERR_UNSUPPORTED;
    vggt::PoolJob job{};
    job.k = k;
    job.v = v;
    job.pos = pos;
    job.k_out = k_out;
    job.k_hat = nullptr;
    job.v_out = v_out;
    job.pos_out = pos_out;
    job.S = S;
    job.T = T;
    job.layout = L;
    job.kd = kv_down;
    job.H = H;
    return to_status(vggt::launch_kv_pool(job, stream));
}

}  // namespace

extern "C" {

int vggt_attn_frame(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                    vggt_bf16* out, int S, int T, int H, int D, int kv_down, cudaStream_t stream) {
    return attn_call(Kind::kFrame, true, q, k, v, pos, out, 1, S, T, H, D, kv_down, nullptr, nullptr,
                     stream);
}

int vggt_attn_global(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                     vggt_bf16* out, int S, int T, int H, int D, int kv_down, cudaStream_t stream) {
    return attn_call(Kind::kGlobal, true, q, k, v, pos, out, 1, S, T, H, D, kv_down, nullptr, nullptr,
                     stream);
}

int vggt_attn_descriptor(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                         const float* pos, vggt_bf16* out, int S, int T, int H, int D, int kv_down,
                         cudaStream_t stream) {
    return attn_call(Kind::kDescriptor, true, q, k, v, pos, out, 1, S, T, H, D, kv_down, nullptr, nullptr,
                     stream);
}

int vggt_attn_frame_ex(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                       vggt_bf16* out, int S, int T, int H, int D, const vggt_qk_norm* norm,
                       cudaStream_t stream) {
    return attn_call(Kind::kFrame, false, q, k, v, pos, out, 1, S, T, H, D, 1, nullptr, norm, stream);
}

int vggt_attn_global_ex(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                        vggt_bf16* out, int S, int T, int H, int D, const vggt_qk_norm* norm,
                        cudaStream_t stream) {
    return attn_call(Kind::kGlobal, false, q, k, v, pos, out, 1, S, T, H, D, 1, nullptr, norm, stream);
}

int vggt_attn_descriptor_ex(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                            const float* pos, vggt_bf16* out, int S, int T, int H, int D, int kv_down,
                            const vggt_frame_layout* layout, const vggt_qk_norm* norm,
                            cudaStream_t stream) {
    return attn_call(Kind::kDescriptor, false, q, k, v, pos, out, 1, S, T, H, D, kv_down, layout, norm,
                     stream);
}

int vggt_attn_global_batch(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                           vggt_bf16* out, int B, int S, int T, int H, int D, const vggt_qk_norm* norm,
                           cudaStream_t stream) {
    return attn_call(Kind::kGlobal, false, q, k, v, pos, out, B, S, T, H, D, 1, nullptr, norm, stream);
}

int vggt_attn_descriptor_batch(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                               vggt_bf16* out, int B, int S, int T, int H, int D, int kv_down,
                               const vggt_frame_layout* layout, const vggt_qk_norm* norm, cudaStream_t stream) {
    return attn_call(Kind::kDescriptor, false, q, k, v, pos, out, B, S, T, H, D, kv_down, layout, norm, stream);
}

int vggt_qk_prologue(const vggt_bf16* x, const float* pos, vggt_bf16* x_hat, int N, int H, int D,
                     cudaStream_t stream) {
    return vggt_qk_prologue_ex(x, pos, x_hat, N, H, D, nullptr, nullptr, stream);
}

int vggt_qk_prologue_ex(const vggt_bf16* x, const float* pos, vggt_bf16* x_hat, int N, int H, int D,
                        const float* ln_weight, const float* ln_bias, cudaStream_t stream) {
    if (N < 0 || H < 0 || D < 0) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    if (N > VGGT_MAX_TOKENS || H > 65535) return VGGT_ERR_SHAPE;
    vggt::LnAffine ln;
    double bound = 0.0;
    if (!make_affine(ln_weight, ln_bias, &ln, &bound)) return VGGT_ERR_UNSUPPORTED;
    if (N == 0 || H == 0) return VGGT_OK;
    if (!x || !pos || !x_hat) return VGGT_ERR_NULL;
    if (!aligned16(x) || !aligned8(pos) || !aligned16(x_hat)) return VGGT_ERR_UNSUPPORTED;
    PrologueJob j{x, pos, x_hat, N, N, ln};
    PrologueJob none{};
    return to_status(vggt::launch_qk_prologue(j, none, H, stream));
}

}  // extern "C"

namespace {

int attn_core_call(const vggt_bf16* q_hat, const vggt_bf16* k_hat, const vggt_bf16* v, vggt_bf16* out, int n_seg,
                   int q_len, int k_len, int H, int D, bool online, cudaStream_t stream) {
    if (n_seg < 0 || q_len < 0 || k_len < 0 || H < 0 || D < 0) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    if (static_cast<long long>(n_seg) * q_len > VGGT_MAX_TOKENS ||
        static_cast<long long>(n_seg) * k_len > VGGT_MAX_TOKENS || H > 65535)
        return VGGT_ERR_SHAPE;
    if (n_seg == 0 || q_len == 0 || k_len == 0 || H == 0) return VGGT_OK;
    if (!q_hat || !k_hat || !v || !out) return VGGT_ERR_NULL;
    if (!aligned16(q_hat) || !aligned16(k_hat) || !aligned16(v) || !aligned16(out))
        return VGGT_ERR_UNSUPPORTED;
    DeviceState* st = status_state();
    if (!st) return VGGT_ERR_CUDA;
    AttnProblem p{q_hat, k_hat, v, out, n_seg, q_len, k_len, H,
                  static_cast<long long>(n_seg) * q_len, static_cast<long long>(n_seg) * k_len};
    p.online = online;
    return to_status(vggt::launch_attention(p, st->status, st->wait_limit, stream));
}

}  // namespace

extern "C" {

int vggt_attn_core(const vggt_bf16* q_hat, const vggt_bf16* k_hat, const vggt_bf16* v,
                   vggt_bf16* out, int n_seg, int q_len, int k_len, int H, int D,
                   cudaStream_t stream) {
    return attn_core_call(q_hat, k_hat, v, out, n_seg, q_len, k_len, H, D, false, stream);
}

int vggt_attn_core_online(const vggt_bf16* q_hat, const vggt_bf16* k_hat, const vggt_bf16* v,
                          vggt_bf16* out, int n_seg, int q_len, int k_len, int H, int D,
                          cudaStream_t stream) {
    return attn_core_call(q_hat, k_hat, v, out, n_seg, q_len, k_len, H, D, true, stream);
}

int vggt_attn_subset(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                     vggt_bf16* out, int S, int T, int n_skip_back, int n_extra, int H, int D, int global,
                     const vggt_qk_norm* norm, cudaStream_t stream) {
    if (S < 0 || T < 1 || H < 0 || D < 0 || n_skip_back < 0 || n_skip_back > T || n_extra < 0)
        return VGGT_ERR_SHAPE;
    if (global != 0 && global != 1) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    if (static_cast<long long>(S) * T + n_extra > VGGT_MAX_TOKENS || H > 65535) return VGGT_ERR_SHAPE;
    Norms norms;
    const int nrc = make_norms(norm, &norms);
    if (nrc != VGGT_OK) return nrc;
    const int keep = T - n_skip_back;
    // rows that take part: the kept tokens of every frame, then (global) the
    // sequence tokens after the frames
    const long long n_frames_rows = static_cast<long long>(S) * keep;
    const long long n = n_frames_rows + (global ? n_extra : 0);
    if (n == 0 || H == 0) return VGGT_OK;
    if (!q || !k || !v || !pos || !out) return VGGT_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned8(pos) || !aligned16(out))
        return VGGT_ERR_UNSUPPORTED;
    DeviceState* st = device_state();
    if (!st) return VGGT_ERR_CUDA;
    vggt::RowMap map;
    if (n_skip_back > 0) {
        map.group = keep;
        map.stride = T;
        map.n_grouped = n_frames_rows;
    }
    const size_t plane = head_plane_bytes(n, H);
    if (norms.precise) {
        // scratch: q_hat fp32 | k_hat terms [H, n, 64] x 2 and, when rows are
        // left out, the gathered values [n, H, 64]
        const size_t ops = precise_bytes(n, n, H);
        void* scratch = nullptr;
        if (cudaMallocFromPoolAsync(&scratch, ops + (n_skip_back > 0 ? plane : 0), st->pool, stream) != cudaSuccess) {
            cudaGetLastError();
            return VGGT_ERR_ALLOC;
        }
        const PreciseOperands po = precise_operands(scratch, n, H);
        const uint16_t* v_use = v;
        int rc = VGGT_OK;
        if (n_skip_back > 0) {
            uint16_t* v_c = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(scratch) + ops);
            rc = to_status(vggt::launch_gather_rows(v, v_c, n, H * VGGT_HEAD_DIM, map, stream));
            v_use = v_c;
        }
        if (rc == VGGT_OK) rc = precise_prologue(q, pos, n, map, k, pos, n, map, po, n, norms, H, stream);
        if (rc == VGGT_OK)
            rc = precise_attention(po, n, v_use, out, global ? 1 : S, global ? static_cast<int>(n) : keep,
                                   global ? static_cast<int>(n) : keep, H, n, map, st, stream);
        cudaFreeAsync(scratch, stream);
        return rc;
    }
    // scratch: q_hat | k_hat [H, n, 64] and, when rows are left out, the
    // gathered values [n, H, 64]
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, (n_skip_back > 0 ? 3 : 2) * plane, st->pool, stream) != cudaSuccess) {
        cudaGetLastError();
        return VGGT_ERR_ALLOC;
    }
    uint16_t* q_hat = static_cast<uint16_t*>(scratch);
    uint16_t* k_hat = q_hat + plane / sizeof(uint16_t);
    const uint16_t* v_use = v;
    int rc = VGGT_OK;
    if (n_skip_back > 0) {
        uint16_t* v_c = k_hat + plane / sizeof(uint16_t);
        rc = to_status(vggt::launch_gather_rows(v, v_c, n, H * VGGT_HEAD_DIM, map, stream));
        v_use = v_c;
    }
    if (rc == VGGT_OK) {
        PrologueJob jq{q, pos, q_hat, static_cast<int>(n), n, norms.q, map};
        PrologueJob jk{k, pos, k_hat, static_cast<int>(n), n, norms.k, map};
        rc = to_status(vggt::launch_qk_prologue(jq, jk, H, stream));
    }
    if (rc == VGGT_OK) {
        AttnProblem p{q_hat, k_hat, v_use, out, global ? 1 : S, global ? static_cast<int>(n) : keep,
                      global ? static_cast<int>(n) : keep, H, n, n, map};
        p.online = norms.online;
        rc = to_status(vggt::launch_attention(p, st->status, st->wait_limit, stream));
    }
    cudaFreeAsync(scratch, stream);
    return rc;
}

}  // extern "C"

namespace {

// The fp32 mode: prologue (q fp32, k split into its bf16 terms), split v,
// attention.
int attn_f32_call(bool global, const float* q, const float* k, const float* v, const float* pos, float* out,
                  int S, int T, int H, int D, const vggt_qk_norm* norm, int terms, cudaStream_t stream) {
    if (terms != 2 && terms != 3) return VGGT_ERR_UNSUPPORTED;
    int rc = check_common(q, k, v, pos, out, S, T, H, D);
    Norms norms;
    if (rc == VGGT_OK || rc == 1) {
        const int nrc = make_norms(norm, &norms);
        if (nrc != VGGT_OK) rc = nrc;
    }
    if (rc != VGGT_OK) return rc == 1 ? VGGT_OK : rc;
    DeviceState* st = device_state();
    if (!st) return VGGT_ERR_CUDA;
    const long long n = static_cast<long long>(S) * T;
    const size_t plane2 = head_plane_bytes(n, H);  // one bf16 [H, n, 64] plane
    // scratch: q_hat fp32 | the k_hat terms | the v terms
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, (2 + 2 * static_cast<size_t>(terms)) * plane2, st->pool, stream) !=
        cudaSuccess) {
        cudaGetLastError();
        return VGGT_ERR_ALLOC;
    }
    float* q_hat = static_cast<float*>(scratch);
    uint16_t* kt[3] = {nullptr, nullptr, nullptr};
    uint16_t* vt[3] = {nullptr, nullptr, nullptr};
    uint16_t* next = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(scratch) + 2 * plane2);
    for (int t = 0; t < terms; ++t, next += plane2 / 2) kt[t] = next;
    for (int t = 0; t < terms; ++t, next += plane2 / 2) vt[t] = next;
    vggt::PrologueJobF32 jq{q, pos, {q_hat, nullptr, nullptr}, static_cast<int>(n), n, norms.q, 0};
    vggt::PrologueJobF32 jk{k, pos, {kt[0], kt[1], kt[2]}, static_cast<int>(n), n, norms.k, terms};
    rc = to_status(vggt::launch_qk_prologue_f32(jq, jk, H, stream));
    if (rc == VGGT_OK) rc = to_status(vggt::launch_split_bf16(v, vt, terms, n * H * VGGT_HEAD_DIM, stream));
    if (rc == VGGT_OK) {
        vggt::AttnProblemF32 p{q_hat, {kt[0], kt[1], kt[2]}, {vt[0], vt[1], vt[2]}, terms, out, global ? 1 : S,
                               global ? static_cast<int>(n) : T, global ? static_cast<int>(n) : T, H, n, n};
        p.online = norms.online;
        rc = to_status(vggt::launch_attention_f32(p, st->status, st->wait_limit, stream));
    }
    cudaFreeAsync(scratch, stream);
    return rc;
}

}  // namespace

extern "C" {

int vggt_attn_frame_f32(const float* q, const float* k, const float* v, const float* pos, float* out, int S, int T,
                        int H, int D, const vggt_qk_norm* norm, int terms, cudaStream_t stream) {
    return attn_f32_call(false, q, k, v, pos, out, S, T, H, D, norm, terms, stream);
}

int vggt_attn_global_f32(const float* q, const float* k, const float* v, const float* pos, float* out, int S, int T,
                         int H, int D, const vggt_qk_norm* norm, int terms, cudaStream_t stream) {
    return attn_f32_call(true, q, k, v, pos, out, S, T, H, D, norm, terms, stream);
}

int vggt_kv_pool_tokens(int T, int kv_down) { return vggt_kv_pool_tokens_ex(T, kv_down, nullptr); }

int vggt_kv_pool_tokens_ex(int T, int kv_down, const vggt_frame_layout* layout) {
    vggt::FrameLayout L{};
    if (T < 1 || kv_down < 1) return VGGT_ERR_SHAPE;
    const int rc = make_layout(layout, T, &L);
    return rc != VGGT_OK ? rc : L.pooled(kv_down);
}

int vggt_kv_pool(const vggt_bf16* k, const vggt_bf16* v, const float* pos, vggt_bf16* k_out,
                 vggt_bf16* v_out, float* pos_out, int S, int T, int H, int D, int kv_down,
                 cudaStream_t stream) {
    return kv_pool_call(k, v, pos, k_out, v_out, pos_out, S, T, H, D, kv_down, nullptr, stream);
}

int vggt_kv_pool_ex(const vggt_bf16* k, const vggt_bf16* v, const float* pos, vggt_bf16* k_out,
                    vggt_bf16* v_out, float* pos_out, int S, int T, int H, int D, int kv_down,
                    const vggt_frame_layout* layout, cudaStream_t stream) {
    return kv_pool_call(k, v, pos, k_out, v_out, pos_out, S, T, H, D, kv_down, layout, stream);
}

int vggt_descriptor_keys(const vggt_bf16* k, const vggt_bf16* v, const float* pos, vggt_bf16* k_hat,
                         vggt_bf16* v_out, float* pos_out, int S, int T, int H, int D, int kv_down,
                         const vggt_frame_layout* layout, const float* ln_weight, const float* ln_bias,
                         cudaStream_t stream) {
    if (S < 0 || T < 1 || H < 0 || D < 0) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    vggt::FrameLayout L{};
    const int lrc = make_layout(layout, T, &L);
    if (lrc != VGGT_OK) return lrc;
    if (kv_down < 1) return VGGT_ERR_SHAPE;
    if (static_cast<long long>(S) * T > VGGT_MAX_TOKENS || H > 65535) return VGGT_ERR_SHAPE;
    Norms norms{};
    double bound = 0.0;
    if (!make_affine(ln_weight, ln_bias, &norms.k, &bound)) return VGGT_ERR_UNSUPPORTED;
    if (S == 0 || H == 0) return VGGT_OK;
    if (!k || !v || !pos || !k_hat || !v_out || !pos_out) return VGGT_ERR_NULL;
    if (!aligned16(k) || !aligned16(v) || !aligned8(pos) || !aligned16(k_hat) || !aligned16(v_out) ||
        !aligned8(pos_out))
        return VGGT_ERR_UNSUPPORTED;
    const long long nk = static_cast<long long>(S) * L.pooled(kv_down);
    return pool_and_prologue(k, v, pos, S, T, L, kv_down, H, k_hat, nk, v_out, pos_out, nullptr, nullptr,
                             0, nullptr, norms, stream);
}
// ------------------------------------------------------------- streaming

}  // extern "C"

struct vggt_desc_cache {
    int device;
    int max_frames, T, H, kv_down, Tk;
    vggt::FrameLayout layout;
    Norms norms;
    long long capacity;  // max_frames * Tk descriptor rows
    int frames;          // frames appended so far
    uint16_t* k_hat;     // [H][capacity][64] normalised pooled keys, head-major
    uint16_t* k_lo;      // precise mode: their second bf16 terms, same layout (else null)
    uint16_t* v;         // [capacity][H][64] pooled values, token-major
    float* pos;          // [capacity][2] cell-mean positions
};

extern "C" {

int vggt_desc_cache_create(vggt_desc_cache** cache, int max_frames, int T, int H, int D,
                           int kv_down) {
    return vggt_desc_cache_create_ex(cache, max_frames, T, H, D, kv_down, nullptr, nullptr);
}

int vggt_desc_cache_create_ex(vggt_desc_cache** cache, int max_frames, int T, int H, int D, int kv_down,
                              const vggt_frame_layout* layout, const vggt_qk_norm* norm) {
    if (!cache) return VGGT_ERR_NULL;
    *cache = nullptr;
    if (max_frames < 1 || T < 1 || H < 1 || kv_down < 1 || H > 65535) return VGGT_ERR_SHAPE;
    if (D != VGGT_HEAD_DIM) return VGGT_ERR_UNSUPPORTED;
    vggt::FrameLayout L{};
    const int lrc = make_layout(layout, T, &L);
    if (lrc != VGGT_OK) return lrc;
    Norms norms;
    const int nrc = make_norms(norm, &norms);
    if (nrc != VGGT_OK) return nrc;
    const int Tk = L.pooled(kv_down);
    const long long capacity = static_cast<long long>(max_frames) * Tk;
    if (capacity > VGGT_MAX_TOKENS || static_cast<long long>(max_frames) * T > VGGT_MAX_TOKENS)
        return VGGT_ERR_SHAPE;
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
    c->Tk = Tk;
    c->layout = L;
    c->norms = norms;
    c->capacity = capacity;
    c->frames = 0;
    const size_t plane = head_plane_bytes(capacity, H);
    const int k_planes = norms.precise ? 2 : 1;
    void* mem = nullptr;
    if (cudaMalloc(&mem, (k_planes + 1) * plane + static_cast<size_t>(capacity) * 2 * sizeof(float)) != cudaSuccess) {
        cudaGetLastError();
        delete c;
        return VGGT_ERR_ALLOC;
    }
    c->k_hat = static_cast<uint16_t*>(mem);
    c->k_lo = norms.precise ? c->k_hat + plane / sizeof(uint16_t) : nullptr;
    c->v = c->k_hat + k_planes * plane / sizeof(uint16_t);
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
    if (cache->norms.precise) {
        // scratch: the chunk's q_hat fp32 [H, C*T, 64]; its descriptors go
        // straight into the cache (keys as two term planes, fp32 means
        // normalised in the pooling pass).
        void* scratch = nullptr;
        if (cudaMallocFromPoolAsync(&scratch, 2 * head_plane_bytes(n_q, H), st->pool, stream) != cudaSuccess) {
            cudaGetLastError();
            return VGGT_ERR_ALLOC;
        }
        const PreciseOperands all{static_cast<float*>(scratch), {cache->k_hat, cache->k_lo}};
        rc = precise_prologue(q, pos, n_q, vggt::RowMap{}, nullptr, nullptr, 0, vggt::RowMap{}, all,
                              cache->capacity, cache->norms, H, stream);
        if (rc == VGGT_OK)
            rc = precise_pool_keys(k, v, pos, C, T, cache->layout, cache->kv_down, H,
                                   cache->k_hat + row0 * VGGT_HEAD_DIM, cache->k_lo + row0 * VGGT_HEAD_DIM,
                                   cache->capacity, cache->v + row0 * H * VGGT_HEAD_DIM, cache->pos + row0 * 2,
                                   cache->norms, stream);
        if (rc == VGGT_OK)
            rc = precise_attention(all, cache->capacity, cache->v, out, 1, static_cast<int>(n_q),
                                   static_cast<int>(row0 + n_new), H, n_q, vggt::RowMap{}, st, stream);
        cudaFreeAsync(scratch, stream);
        if (rc == VGGT_OK) cache->frames += C;
        return rc;
    }
    // Scratch: the chunk's q_hat [H, C*T, 64].
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, head_plane_bytes(n_q, H), st->pool, stream) != cudaSuccess) {
        cudaGetLastError();
        return VGGT_ERR_ALLOC;
    }
    uint16_t* q_hat = static_cast<uint16_t*>(scratch);
    // 1. The chunk's queries through the prologue, and its descriptors
    //    straight into the cache (values and positions at row0, normalised
    //    keys at row0 of every head's plane).
    rc = pool_and_prologue(k, v, pos, C, T, cache->layout, cache->kv_down, H,
                           cache->k_hat + row0 * VGGT_HEAD_DIM, cache->capacity,
                           cache->v + row0 * H * VGGT_HEAD_DIM, cache->pos + row0 * 2, q, pos, n_q, q_hat,
                           cache->norms, stream);
    // 2. Every query of the chunk attends to every cached descriptor.
    if (rc == VGGT_OK) {
        AttnProblem p{q_hat, cache->k_hat, cache->v, out, 1, static_cast<int>(n_q),
                      static_cast<int>(row0 + n_new), H, n_q, cache->capacity};
        p.online = cache->norms.online;
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

int vggt_scratch_pool_info(int* exists, unsigned long long* reserved) {
    if (!exists || !reserved) return VGGT_ERR_NULL;
    *exists = 0;
    *reserved = 0;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VGGT_ERR_CUDA;
    DeviceState& st = g_dev[dev];
    if (!st.ready.load(std::memory_order_acquire)) return VGGT_OK;
    uint64_t bytes = 0;
    if (cudaMemPoolGetAttribute(st.pool, cudaMemPoolAttrReservedMemCurrent, &bytes) != cudaSuccess) {
        cudaGetLastError();
        return VGGT_ERR_CUDA;
    }
    *exists = 1;
    *reserved = static_cast<unsigned long long>(bytes);
    return VGGT_OK;
}

int vggt_get_device_status(cudaStream_t stream) {
    DeviceState* st = status_state();
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
                   "positions 8), the current device the cache's, and a QK LayerNorm affine finite";
        case VGGT_ERR_SHAPE: return "VGGT_ERR_SHAPE: invalid sizes";
        case VGGT_ERR_ALLOC: return "VGGT_ERR_ALLOC: scratch allocation failed";
        case VGGT_ERR_CUDA: return "VGGT_ERR_CUDA: CUDA call or launch failed";
        case VGGT_ERR_TIMEOUT: return "VGGT_ERR_TIMEOUT: a bounded device wait ran out";
        case VGGT_ERR_RANGE:
            return "VGGT_ERR_RANGE: an attention row sum was not a positive finite number "
                   "(q_hat/k_hat outside vggt_attn_core's norm bound; vggt_attn_core_online takes any)";
        default: return "unknown vggt_status";
    }
}

long long vggt_set_wait_limit(long long cycles) {
    DeviceState* st = status_state();
    if (!st) return -1;
    return st->wait_limit.exchange(cycles < 1 ? kDefaultWaitLimit : cycles);
}

int vggt_debug_wait_timeout(cudaStream_t stream) {
    DeviceState* st = status_state();
    if (!st) return VGGT_ERR_CUDA;
    return to_status(vggt::launch_wait_probe(st->status, st->wait_limit, stream));
}

}  // extern "C"
