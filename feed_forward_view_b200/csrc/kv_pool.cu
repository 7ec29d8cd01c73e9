// kv_pool.cu -- per-frame K/V descriptors for compressed-descriptor attention
// (FlashVGGT README: global attention over a compact per-frame descriptor set
// obtained by spatially resampling keys and values; --kv_downfactor 4), and
// the same pass fused with the key prologue.
//
// A frame of T = n_front + gh*gw + n_back tokens becomes
// Tk = n_front + nch*ncw + n_back tokens, nch = ceil(gh/kd), ncw = ceil(gw/kd):
//   tokens 0 .. n_front-1 (VGGT-1B: camera + 4 registers) are copied bit for bit;
//   token n_front + cr*ncw + cc is cell (cr, cc): patches rows
//   [cr*kd, min(cr*kd+kd, gh)) x cols [cc*kd, min(cc*kd+kd, gw)). Per channel
//   the members are summed in float32 in row-major order, the sum is divided
//   in float32 (IEEE, round to nearest) by the member count, and the quotient
//   is rounded to bf16 (nearest, ties to even). The position is the same
//   float32 mean of member positions;
//   the n_back trailing tokens (the VGGT-Omega page appends its registers
//   after the patches) are copied bit for bit after the cells.
// The fixed order and correctly rounded division make the result bit-exact
// (a power-of-two count divides as an exact product with its reciprocal).
//
// Fused mode: instead of writing the pooled keys, the block normalises each
// pooled key head (LayerNorm + optional affine) and rotates it at the pooled
// position with the prologue's own arithmetic (prologue.cuh), writing the
// head-major k_hat the attention kernel reads. The pooled keys never reach
// memory, and the result is bit-identical to pooling then running the
// prologue. Precise fused mode (calls whose QK LayerNorm affine needs more
// score precision than bf16 keys give) skips the bf16 rounding of the pooled
// keys, normalises the fp32 means and writes k_hat as two bf16 terms.
//
// Memory-bound: every input byte of K and V is read once, the pooled tokens
// are written once. One block per pooled token: 128 threads pool the values,
// 16 heads per pass (8 threads per head, one 16-byte piece per member each);
// the keys take 128 threads laid out the same way in plain mode, or 64
// threads in fused mode (4 threads per head, two 16-byte pieces per member
// each) -- so every member is read with coalesced 128-bit accesses to its
// 2 KB rows of K and V, both in flight together. The sums use packed two-lane
// float32 adds (the kernel is otherwise close to instruction-bound).
#include "pdl.cuh"
#include "prologue.cuh"
#include "sm100.cuh"

namespace vggt {
namespace {

constexpr int kBatch = 8;  // member loads a value thread keeps in flight

// Which source tokens pooled token i of a frame averages: a single copied
// token (src0 + first, copy == true), or the cell rows [r0, r1) x cols
// [c0, c1) of the grid starting at token src0 + n_front.
struct Sources {
    bool copy;
    int first;
    int r0, r1, c0, c1;
};

__device__ __forceinline__ Sources sources_of(const FrameLayout& L, int kd, int i) {
    Sources s{};
    const int ncw = (L.grid_w + kd - 1) / kd;
    const int nch = (L.grid_h + kd - 1) / kd;
    const int ncells = nch * ncw;
    if (i < L.n_front) {
        s.copy = true;
        s.first = i;
    } else if (i < L.n_front + ncells) {
        const int cell = i - L.n_front;
        const int cr = cell / ncw, cc = cell % ncw;
        s.copy = false;
        s.r0 = cr * kd;
        s.r1 = min(s.r0 + kd, L.grid_h);
        s.c0 = cc * kd;
        s.c1 = min(s.c0 + kd, L.grid_w);
    } else {
        s.copy = true;
        s.first = L.n_front + L.grid_h * L.grid_w + (i - L.n_front - ncells);
    }
    return s;
}

// One warp (all lanes): the pooled position of the block's token -- copied,
// or the float32 mean of the members' positions summed in row-major order.
// Lane m loads member m of each batch of 32 (all loads in flight at once),
// then the sums run in member order through shuffles, so the bits are those
// of a plain sequential loop. The result is valid in every lane.
__device__ __forceinline__ float2 pooled_position(const PoolJob& job, const Sources src, size_t src0,
                                                  size_t grid0, float count, int lane) {
    const float2* pos = reinterpret_cast<const float2*>(job.pos);
    if (src.copy) return pos[src0 + src.first];
    const int w = src.c1 - src.c0;
    const int n = (src.r1 - src.r0) * w;
    float pr = 0.f, pc = 0.f;
    for (int b = 0; b < n; b += 32) {
        const int m = b + lane;
        float2 p = make_float2(0.f, 0.f);
        if (m < n) p = pos[grid0 + static_cast<size_t>(src.r0 + m / w) * job.layout.grid_w + src.c0 + m % w];
        const int cnt = min(32, n - b);
        for (int j = 0; j < cnt; ++j) {
            pr = __fadd_rn(pr, __shfl_sync(0xFFFFFFFFu, p.x, j));
            pc = __fadd_rn(pc, __shfl_sync(0xFFFFFFFFu, p.y, j));
        }
    }
    return make_float2(__fdiv_rn(pr, count), __fdiv_rn(pc, count));
}

// The member sums of one thread: kPieces 16-byte pieces per member (8 dims
// each) at byte offsets off[0..kPieces) of every member row, summed in member
// order (row-major over the cell) into packed fp32 pairs acc[4 * piece + e],
// kB members' loads in flight before their sums; then divided by the member
// count (IEEE, or the exact product with the reciprocal of a power of two).
// p: the first member's row (+ the head's offset).
template <int kPieces, int kB>
__device__ __forceinline__ void member_means(const uint8_t* p, const int (&off)[kPieces], size_t tok_b,
                                             size_t row_skip, int cw, int n, bool pow2, float count,
                                             uint64_t (&acc)[4 * kPieces]) {
#pragma unroll
    for (int e = 0; e < 4 * kPieces; ++e) acc[e] = 0;
    int c = 0;
    for (int m0 = 0; m0 < n; m0 += kB) {
        uint4 w[kB][kPieces];
#pragma unroll
        for (int j = 0; j < kB; ++j) {
            if (m0 + j < n) {
#pragma unroll
                for (int q = 0; q < kPieces; ++q) w[j][q] = __ldg(reinterpret_cast<const uint4*>(p + off[q]));
                p += tok_b;
                if (++c == cw) {
                    c = 0;
                    p += row_skip;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kB; ++j) {
            if (m0 + j < n) {
#pragma unroll
                for (int q = 0; q < kPieces; ++q) {
                    acc[4 * q + 0] = f2_add(acc[4 * q + 0], u2_pack(w[j][q].x << 16, w[j][q].x & 0xFFFF0000u));
                    acc[4 * q + 1] = f2_add(acc[4 * q + 1], u2_pack(w[j][q].y << 16, w[j][q].y & 0xFFFF0000u));
                    acc[4 * q + 2] = f2_add(acc[4 * q + 2], u2_pack(w[j][q].z << 16, w[j][q].z & 0xFFFF0000u));
                    acc[4 * q + 3] = f2_add(acc[4 * q + 3], u2_pack(w[j][q].w << 16, w[j][q].w & 0xFFFF0000u));
                }
            }
        }
    }
    if (pow2) {
        const uint64_t inv2 = f2_pack(1.0f / count, 1.0f / count);
#pragma unroll
        for (int e = 0; e < 4 * kPieces; ++e) acc[e] = f2_mul(acc[e], inv2);
    } else {
#pragma unroll
        for (int e = 0; e < 4 * kPieces; ++e) {
            float x, y;
            f2_unpack(acc[e], x, y);
            acc[e] = f2_pack(__fdiv_rn(x, count), __fdiv_rn(y, count));
        }
    }
}

// 4 consecutive values of a 16-byte bf16 piece (half 0: the first 4, half 1:
// the last 4), widened.
__device__ __forceinline__ void piece_half(uint4 w, int half, float (&x)[4]) {
    const uint32_t u = half ? w.z : w.x, v = half ? w.w : w.y;
    x[0] = prologue::bf16_lo(u);
    x[1] = prologue::bf16_hi(u);
    x[2] = prologue::bf16_lo(v);
    x[3] = prologue::bf16_hi(v);
}
// 4 consecutive means (pairs acc[first], acc[first + 1]), as stored (bf16)
// or (kPrecise) as they are.
template <bool kPrecise>
__device__ __forceinline__ void means4(const uint64_t (&acc)[8], int first, float (&x)[4]) {
    f2_unpack(acc[first], x[0], x[1]);
    f2_unpack(acc[first + 1], x[2], x[3]);
    if (!kPrecise) {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
    }
}

// kFused: keys normalised and rotated into k_hat (else pooled into k_out);
// kAffine: the key LayerNorm has an affine; kPrecise (fused only): fp32 means
// into the prologue, two-term k_hat. Separate instantiations keep the plain
// pooling at its register count; at most 64 registers a thread (four plain
// blocks or five fused ones per SM) measured fastest: occupancy decides this
// memory-bound kernel more than the few registers it then spills.
//
// Plain mode (256 threads): warps 0-3 pool the values, warps 4-7 the keys,
// 16 heads per pass, 8 threads per head, one 16-byte piece (8 dims) per
// member, kBatch members' loads in flight. Fused mode (128 threads): warps
// 0-1 pool the values, 4 threads per head with two 16-byte pieces (16 dims)
// per member and kBatch / 2 members in flight; warps 2-3 the keys, 4 threads
// per head holding the prologue's two units (dims d1..d1+7 and d1+16..d1+23,
// two 16-byte pieces per member, kBatch / 2 members in flight), which go on
// from their means to the prologue arithmetic (norm_rotate2) with no
// exchange of values. (The key threads carry the longer path -- their means
// and then the prologue -- so the two groups are given the same number of
// warps; with four value warps beside two key warps, the value warps idled
// half the block and five blocks fitted an SM, against eight now.) A thread
// walks its cell's members in row-major order with a pointer; the sums keep
// the member order. Warp 0 first gathers the pooled position; in fused mode
// it hands it to the key warps through named barrier 1 (the value warps never
// wait).
template <bool kFused>
constexpr int pool_threads() {
    return kFused ? 128 : 256;
}

template <bool kFused, bool kAffine, bool kPrecise>
__global__ void __launch_bounds__(pool_threads<kFused>(), kFused ? 8 : 4)
kv_pool_kernel(const __grid_constant__ PoolJob job, FreqTable freq) {
    griddep_wait();  // before any global memory access (pdl.cuh)
    __shared__ float2 pooled_pos;
    __shared__ __align__(16) prologue::SmemAffine sk;
    constexpr int kValueThreads = kFused ? 64 : 128;
    constexpr int kKeyThreads = pool_threads<kFused>() - kValueThreads;
    constexpr uint32_t kKeyBar = 1, kKeyBarThreads = 32 + kKeyThreads;  // warp 0 + the key warps
    constexpr int kHeadsPerPass = 16;
    static_assert(kValueThreads / (kFused ? 4 : 8) == kHeadsPerPass && (!kFused || kKeyThreads / 4 == kHeadsPerPass),
                  "each group covers kHeadsPerPass heads per pass");

    const FrameLayout& L = job.layout;
    const int lane = threadIdx.x & 31;
    const bool keys = threadIdx.x >= kValueThreads;
    const int t = keys ? threadIdx.x - kValueThreads : threadIdx.x;  // thread within its group
    const int Tk = L.pooled(job.kd);
    const int s = blockIdx.x / Tk;  // frame
    const int i = blockIdx.x % Tk;  // pooled token within the frame
    const size_t src0 = static_cast<size_t>(s) * job.T;
    const size_t dst = static_cast<size_t>(s) * Tk + i;
    const size_t grid0 = src0 + L.n_front;
    const Sources src = sources_of(L, job.kd, i);
    const int cw = src.c1 - src.c0;
    const int n = src.copy ? 1 : (src.r1 - src.r0) * cw;  // member tokens
    const float count = static_cast<float>(n);
    // a power-of-two count divides exactly as a product with its reciprocal
    const bool pow2 = (n & (n - 1)) == 0;
    const size_t tok = static_cast<size_t>(job.H) * kHeadDim;  // elements per token
    const size_t tok_b = tok * 2;                              // bytes per token

    const float* aff = nullptr;
    if (kAffine && keys) {
        for (int e = t; e < 2 * kHeadDim; e += kKeyThreads)
            sk.v[e] = e < kHeadDim ? job.k_ln.gamma[e] : job.k_ln.beta[e - kHeadDim];
        aff = sk.v;
    }
    if (threadIdx.x < 32) {
        const float2 p = pooled_position(job, src, src0, grid0, count, lane);
        if (lane == 0) {
            reinterpret_cast<float2*>(job.pos_out)[dst] = p;
            pooled_pos = p;
        }
        if (kFused) named_bar_arrive(kKeyBar, kKeyBarThreads);
    }

    const uint8_t* in = reinterpret_cast<const uint8_t*>(keys ? job.k : job.v);
    const size_t row_skip = static_cast<size_t>(L.grid_w - cw) * tok_b;
    const uint8_t* first = in + (grid0 + static_cast<size_t>(src.r0) * L.grid_w + src.c0) * tok_b;

    if (!kFused || !keys) {
        // ---- values (and plain keys): dims dv .. dv + 8 * kPieces - 1 of head h,
        // token-major out
        constexpr int kShift = kFused ? 2 : 3;    // log2 of the threads per head
        constexpr int kPieces = 8 >> kShift;      // 16-byte pieces (8 dims) per member
        const int dv = 8 * kPieces * (t & ((1 << kShift) - 1));
        uint16_t* out_base = keys ? job.k_out : job.v_out;
        for (int h0 = 0; h0 < job.H; h0 += kHeadsPerPass) {
            const int h = h0 + (t >> kShift);
            if (h >= job.H) continue;
            const size_t hoff = static_cast<size_t>(h) * kHeadDim * 2;
            uint4 o[kPieces];
            if (src.copy) {
#pragma unroll
                for (int q = 0; q < kPieces; ++q)
                    o[q] = __ldg(reinterpret_cast<const uint4*>(in + (src0 + src.first) * tok_b + hoff + 2 * (dv + 8 * q)));
            } else {
                uint64_t acc[4 * kPieces];
                int off[kPieces];
#pragma unroll
                for (int q = 0; q < kPieces; ++q) off[q] = 2 * (dv + 8 * q);
                member_means<kPieces, kBatch / kPieces>(first + hoff, off, tok_b, row_skip, cw, n, pow2, count, acc);
#pragma unroll
                for (int q = 0; q < kPieces; ++q) {
                    float m[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) f2_unpack(acc[4 * q + e], m[2 * e], m[2 * e + 1]);
                    o[q] = make_uint4(prologue::pack2(m[0], m[1]), prologue::pack2(m[2], m[3]),
                                      prologue::pack2(m[4], m[5]), prologue::pack2(m[6], m[7]));
                }
            }
#pragma unroll
            for (int q = 0; q < kPieces; ++q)
                *reinterpret_cast<uint4*>(out_base + dst * tok + static_cast<size_t>(h) * kHeadDim + dv + 8 * q) = o[q];
        }
        griddep_launch_dependents();
        return;
    }

    // ---- fused keys: units a (dims d1..d1+3, d1+16..d1+19) and b (d1+4..,
    // d1+20..) of head h, pooled, then normalised and rotated at the pooled
    // position
    const int sub = lane & 3;
    const int d1 = (sub >> 1) * 32 + 8 * (sub & 1);
    float sa[4], ca[4], sb[4], cb[4];
    for (int h0 = 0; h0 < job.H; h0 += kHeadsPerPass) {
        const int h = h0 + (t >> 2);
        const bool live = h < job.H;
        float a1[4] = {0.f, 0.f, 0.f, 0.f}, a2[4] = {0.f, 0.f, 0.f, 0.f};
        float b1[4] = {0.f, 0.f, 0.f, 0.f}, b2[4] = {0.f, 0.f, 0.f, 0.f};
        if (live) {
            const size_t hoff = static_cast<size_t>(h) * kHeadDim * 2;
            if (src.copy) {
                const uint8_t* p = in + (src0 + src.first) * tok_b + hoff;
                const uint4 lo = __ldg(reinterpret_cast<const uint4*>(p + 2 * d1));
                const uint4 hi = __ldg(reinterpret_cast<const uint4*>(p + 2 * (d1 + 16)));
                piece_half(lo, 0, a1);
                piece_half(lo, 1, b1);
                piece_half(hi, 0, a2);
                piece_half(hi, 1, b2);
            } else {
                uint64_t acc[8];
                const int off[2] = {2 * d1, 2 * (d1 + 16)};
                member_means<2, kBatch / 2>(first + hoff, off, tok_b, row_skip, cw, n, pow2, count, acc);
                // the pooled keys as stored (bf16; precise mode: the fp32 means)
                means4<kPrecise>(acc, 0, a1);
                means4<kPrecise>(acc, 2, b1);
                means4<kPrecise>(acc, 4, a2);
                means4<kPrecise>(acc, 6, b2);
            }
        }
        if (h0 == 0) {
            named_bar_sync(kKeyBar, kKeyBarThreads);  // pooled_pos and the staged affine
            prologue::token_angles2(pooled_pos, lane, prologue::lane_freq(freq, lane), sa, ca, sb, cb);
        }
        float oa1[4], oa2[4], ob1[4], ob2[4];
        prologue::norm_rotate2<kAffine, false>(a1, a2, b1, b2, aff, sa, ca, sb, cb, d1, oa1, oa2, ob1, ob2);
        if (!live) continue;
        uint16_t* out = job.k_hat + (static_cast<size_t>(h) * job.k_hat_stride + dst) * kHeadDim;
        if constexpr (kPrecise) {
            uint16_t* lo = job.k_hat_lo + (static_cast<size_t>(h) * job.k_hat_stride + dst) * kHeadDim;
            prologue::store_two_terms(out, lo, d1, oa1, oa2);
            prologue::store_two_terms(out, lo, d1 + 4, ob1, ob2);
        } else {
            *reinterpret_cast<uint4*>(out + d1) =
                make_uint4(prologue::pack2(oa1[0], oa1[1]), prologue::pack2(oa1[2], oa1[3]),
                           prologue::pack2(ob1[0], ob1[1]), prologue::pack2(ob1[2], ob1[3]));
            *reinterpret_cast<uint4*>(out + d1 + 16) =
                make_uint4(prologue::pack2(oa2[0], oa2[1]), prologue::pack2(oa2[2], oa2[3]),
                           prologue::pack2(ob2[0], ob2[1]), prologue::pack2(ob2[2], ob2[3]));
        }
    }
    griddep_launch_dependents();
}

template <bool kFused, bool kAffine, bool kPrecise = false>
cudaError_t launch_pool_kernel(const PoolJob& job, unsigned blocks, cudaStream_t stream) {
    return launch_pdl(kv_pool_kernel<kFused, kAffine, kPrecise>, dim3(blocks), dim3(pool_threads<kFused>()), 0, stream,
                      job, rope_freq_table());
}

}  // namespace

cudaError_t launch_kv_pool(const PoolJob& job, cudaStream_t stream) {
    const int Tk = job.layout.pooled(job.kd);
    const long long blocks = (job.S > 0 && job.H > 0) ? static_cast<long long>(job.S) * Tk : 0;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    const unsigned b = static_cast<unsigned>(blocks);
    if (job.k_hat == nullptr) return launch_pool_kernel<false, false>(job, b, stream);
    if (job.k_hat_lo != nullptr)
        return job.k_ln.on ? launch_pool_kernel<true, true, true>(job, b, stream)
                           : launch_pool_kernel<true, false, true>(job, b, stream);
    return job.k_ln.on ? launch_pool_kernel<true, true>(job, b, stream)
                       : launch_pool_kernel<true, false>(job, b, stream);
}

}  // namespace vggt
