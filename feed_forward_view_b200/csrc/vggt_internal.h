// vggt_internal.h -- host-side launchers shared by the C ABI (abi.cu) and the
// kernel translation units. Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime_api.h>

namespace vggt {

constexpr int kNSpecial = 5;
constexpr int kHeadDim = 64;

// Bits of the device status word.
constexpr int kStatusTimeout = 1;  // a bounded device wait ran out
constexpr int kStatusRange = 2;    // an attention row sum was not a positive finite number

// One tensor to normalise and rotate: x [n, H, 64] token-major in, positions
// pos [n, 2] (row, col); out head-major: row t of head h goes to
// x_hat + (h * out_stride + t) * 64 (out_stride = n for a [H, n, 64] array;
// larger to write n rows into a bigger head-major array at x_hat's row).
struct PrologueJob {
    const uint16_t* x;
    const float* pos;
    uint16_t* x_hat;
    int n;
    long long out_stride;
};

// LayerNorm (eps 1e-5, no affine) + 2D RoPE (base 100) over one or two jobs in
// a single launch. Returns the launch's cudaError_t.
cudaError_t launch_qk_prologue(const PrologueJob& a, const PrologueJob& b, int H,
                               cudaStream_t stream);

// Ceil-mode kd x kd average pooling of the patch grid of every frame, special
// tokens copied. k,v [S*T, H, 64] -> [S*Tk, H, 64]; pos [S*T,2] -> [S*Tk,2].
cudaError_t launch_kv_pool(const uint16_t* k, const uint16_t* v, const float* pos,
                           uint16_t* k_out, uint16_t* v_out, float* pos_out,
                           int S, int T, int g, int kd, int H, cudaStream_t stream);

// Attention over segments: segment s has queries rows [s*q_len, (s+1)*q_len)
// of q_hat and keys rows [s*k_len, (s+1)*k_len) of k_hat / v.
//   q_hat and k_hat head-major: row r of head h at q_hat + (h * q_stride + r)
//   * 64 (likewise k_hat with k_stride); q_stride >= n_seg*q_len, k_stride >=
//   n_seg*k_len (equal for plain [H, n, 64] arrays);
//   v [n_seg*k_len, H, 64] and out [n_seg*q_len, H, 64] token-major.
struct AttnProblem {
    const uint16_t* q_hat;
    const uint16_t* k_hat;
    const uint16_t* v;
    uint16_t* out;
    int n_seg;
    int q_len;
    int k_len;
    int H;
    long long q_stride;
    long long k_stride;
};

// Returns cudaSuccess, or an error from tensor-map encoding or the launch.
cudaError_t launch_attention(const AttnProblem& p, int* status, long long wait_limit,
                             cudaStream_t stream);

// Device address of the library's device status word and the current
// bounded-wait limit, for the current device; false if the lookup failed.
bool device_status_word(int** status, long long* wait_limit);

// A one-thread kernel that waits on a barrier nothing completes.
cudaError_t launch_wait_probe(int* status, long long wait_limit, cudaStream_t stream);

}  // namespace vggt
