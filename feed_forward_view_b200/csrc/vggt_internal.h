// vggt_internal.h -- host-side launchers shared by the C ABI (abi.cu) and the
// kernel translation units. Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime_api.h>

#ifdef __CUDACC__
#define VGGT_HD __host__ __device__
#else
#define VGGT_HD
#endif

namespace vggt {

constexpr int kNSpecial = 5;
constexpr int kHeadDim = 64;

// Bits of the device status word.
constexpr int kStatusTimeout = 1;  // a bounded device wait ran out
constexpr int kStatusRange = 2;    // an attention row sum was not a positive finite number

// Compact row c -> original token row. Identity when group == 0; otherwise
// the first n_grouped compact rows come in groups of `group` rows whose
// originals start `stride` rows apart (row c at (c / group) * stride + c %
// group), and the rows from n_grouped on follow the last group's stride
// contiguously. Used for calls where a frame's trailing tokens take no part:
// group = kept tokens per frame, stride = T.
struct RowMap {
    long long group = 0, stride = 0, n_grouped = 0;
};
VGGT_HD inline long long map_row(const RowMap& m, long long c) {
    if (m.group == 0) return c;
    if (c < m.n_grouped) return (c / m.group) * m.stride + c % m.group;
    return (m.n_grouped / m.group) * m.stride + (c - m.n_grouped);
}

// RoPE frequencies 100^(-j/16), j = 0..15, in fp32, passed by value.
struct FreqTable {
    float f[16];
};
FreqTable rope_freq_table();

// Optional per-dim scale and shift after a QK LayerNorm (shared by the
// heads), passed by value; on == 0 means none.
struct LnAffine {
    float gamma[kHeadDim];
    float beta[kHeadDim];
    int on;
};

// One tensor to normalise and rotate: x [., H, 64] token-major in, positions
// pos [., 2] (row, col); n rows out, head-major: row t of head h goes to
// x_hat + (h * out_stride + t) * 64 (out_stride = n for a [H, n, 64] array;
// larger to write n rows into a bigger head-major array at x_hat's row). Row
// t reads token map_row(in_map, t) of x and pos (identity by default).
struct PrologueJob {
    const uint16_t* x;
    const float* pos;
    uint16_t* x_hat;
    int n;
    long long out_stride;
    LnAffine ln;
    RowMap in_map;
};

// LayerNorm (eps 1e-5, optional affine) + 2D RoPE (base 100) over one or two
// jobs in a single launch. Returns the launch's cudaError_t.
cudaError_t launch_qk_prologue(const PrologueJob& a, const PrologueJob& b, int H,
                               cudaStream_t stream);

// Token layout of one frame: n_front special tokens, a grid_h x grid_w patch
// grid in row-major order, n_back trailing tokens.
struct FrameLayout {
    int n_front, grid_h, grid_w, n_back;
    VGGT_HD int tokens() const { return n_front + grid_h * grid_w + n_back; }
    // tokens per pooled frame for kd x kd ceil-mode cells
    VGGT_HD int pooled(int kd) const {
        const int nch = grid_h > 0 ? (grid_h + kd - 1) / kd : 0;
        const int ncw = grid_w > 0 ? (grid_w + kd - 1) / kd : 0;
        return n_front + nch * ncw + n_back;
    }
};

// The prologue with fp32 or term-split results (the fp32 mode, and bf16 calls
// whose affine needs more score precision). One tensor x [., H, 64] (fp32, or
// bf16 when x_bf16; positions pos [., 2]) through the prologue; n rows out,
// head-major: row t of head h at (h * out_stride + t) * 64, read from token
// map_row(in_map, t) of x and pos. terms == 0: fp32 results to out[0];
// terms == 2 or 3: that many bf16 terms (y_0 = bf16(y), y_1 = bf16(y - y_0),
// y_2 = bf16(y - y_0 - y_1)) to out[0..]. Both jobs of a launch take the same
// input type.
struct PrologueJobF32 {
    const void* x;
    const float* pos;
    void* out[3];
    int n;
    long long out_stride;
    LnAffine ln;
    int terms;
    bool x_bf16 = false;
    RowMap in_map;
};
cudaError_t launch_qk_prologue_f32(const PrologueJobF32& a, const PrologueJobF32& b, int H,
                                   cudaStream_t stream);
// The bf16 terms (2 or 3) of n fp32 values (n a multiple of 4), same layout.
cudaError_t launch_split_bf16(const float* x, uint16_t* const (&out)[3], int terms, long long n,
                              cudaStream_t stream);

// Attention on term-split operands: segments as in AttnProblem; q_hat fp32
// head-major (plane stride q_stride), the bf16 terms of k_hat head-major
// (plane stride k_stride) and of v [n_seg*k_len, H, 64].
//   terms == terms_pv (2 or 3): the fp32 mode; out fp32 [n_seg*q_len, H, 64].
//   terms == 2, terms_pv == 1: bf16 calls that need precise scores; q_hat and
//   k_hat in two terms, P and v in one (v[0] = the bf16 v), out bf16, online
//   softmax required.
// Query row r is stored at output row map_row(out_map, r).
struct AttnProblemF32 {
    const float* q_hat;
    const uint16_t* k[3];
    const uint16_t* v[3];
    int terms;
    void* out;
    int n_seg;
    int q_len;
    int k_len;
    int H;
    long long q_stride;
    long long k_stride;
    bool online = false;  // running row maximum, as in AttnProblem
    int terms_pv = 0;     // 0: the same as terms
    RowMap out_map;
};
cudaError_t launch_attention_f32(const AttnProblemF32& p, int* status, long long wait_limit,
                                 cudaStream_t stream);

// dst row c = src row map_row(m, c) for c < n; rows of `row_elems` bf16
// values (a multiple of 8).
cudaError_t launch_gather_rows(const uint16_t* src, uint16_t* dst, long long n, int row_elems,
                               const RowMap& m, cudaStream_t stream);

// Ceil-mode kd x kd average pooling of the patch grid of every frame, special
// tokens copied; pooled frame = front specials, cells row-major, trailing
// tokens. v [S*T, H, 64] -> v_out [S*Tk, H, 64]; pos [S*T,2] -> pos_out
// [S*Tk,2]. Keys either pooled the same way into k_out (k_hat == nullptr), or
// (k_out == nullptr) pooled, normalised (k_ln) and rotated at their pooled
// position, and written head-major: pooled row r of head h at
// k_hat + (h * k_hat_stride + r) * 64. With k_hat_lo set as well (precise
// mode), the pooled keys stay fp32 means (no bf16 rounding) before the
// prologue, whose results go out as two bf16 terms: k_hat and k_hat_lo.
struct PoolJob {
    const uint16_t* k;
    const uint16_t* v;
    const float* pos;
    uint16_t* k_out;
    uint16_t* k_hat;
    long long k_hat_stride;
    uint16_t* k_hat_lo = nullptr;
    uint16_t* v_out;
    float* pos_out;
    int S, T;
    FrameLayout layout;
    int kd, H;
    LnAffine k_ln;
};
cudaError_t launch_kv_pool(const PoolJob& job, cudaStream_t stream);

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
    RowMap out_map;  // output row of query row r: map_row(out_map, r)
    // Softmax with a running row maximum (any finite inputs) instead of the
    // maximum-free form, which needs |score| * log2(e) within about 2^6.
    bool online = false;
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
