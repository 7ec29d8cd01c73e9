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
// are written once. One 256-thread block per pooled token: 128 threads pool
// the values, 128 the keys, 16 heads per pass (8 threads per head). Per
// member token a value thread loads its head's 16 bytes (dims 8*(t%8) ..); a
// key thread loads the same in plain mode, or the prologue's two 8-byte
// pieces (dims d1.., d1+16..) in fused mode -- so every member is read with
// fully coalesced 2 KB rows of K and V, both in flight together. The sums
// use packed two-lane float32 adds (the kernel is otherwise close to
// instruction-bound).
#include "prologue.cuh"
#include "sm100.cuh"

namespace vggt {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 8;  // member loads a thread keeps in flight

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

// 8 bf16 values (w) added to 4 float32 pairs, two adds per instruction
__device__ __forceinline__ void add8x2(uint64_t (&acc)[4], uint2 lo, uint2 hi) {
    acc[0] = f2_add(acc[0], u2_pack(lo.x << 16, lo.x & 0xFFFF0000u));
    acc[1] = f2_add(acc[1], u2_pack(lo.y << 16, lo.y & 0xFFFF0000u));
    acc[2] = f2_add(acc[2], u2_pack(hi.x << 16, hi.x & 0xFFFF0000u));
    acc[3] = f2_add(acc[3], u2_pack(hi.y << 16, hi.y & 0xFFFF0000u));
}

// kFused: keys normalised and rotated into k_hat (else pooled into k_out);
// kAffine: the key LayerNorm has an affine; kPrecise (fused only): fp32 means
// into the prologue, two-term k_hat. Separate instantiations keep the
// plain pooling at its register count. Four resident blocks per SM (<= 64
// registers a thread) measured fastest: occupancy decides this memory-bound
// kernel more than the few registers it then spills.
//
// 256 threads: warps 0-3 pool the values, warps 4-7 the keys, 16 heads per
// pass (8 threads per head). A thread walks its cell's members in row-major
// order with a pointer, kBatch member loads in flight before the sums (which
// keep the member order). Warp 0 first gathers the pooled position; in fused
// mode it hands it to the key warps through named barrier 1 (the value warps
// never wait).
template <bool kFused, bool kAffine, bool kPrecise>
__global__ void __launch_bounds__(kThreads, 4)
kv_pool_kernel(const __grid_constant__ PoolJob job, FreqTable freq) {
    __shared__ float2 pooled_pos;
    __shared__ __align__(16) prologue::SmemAffine sk;
    constexpr uint32_t kKeyBar = 1, kKeyBarThreads = 32 + kThreads / 2;  // warp 0 + the key warps

    const FrameLayout& L = job.layout;
    const int lane = threadIdx.x & 31;
    const bool keys = threadIdx.x >= kThreads / 2;
    const int t = threadIdx.x & (kThreads / 2 - 1);  // thread within its half
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
    const uint64_t inv2 = f2_pack(1.0f / count, 1.0f / count);
    const size_t tok = static_cast<size_t>(job.H) * kHeadDim;  // elements per token
    const size_t tok_b = tok * 2;                              // bytes per token

    const float* aff = nullptr;
    if (kAffine && keys) {
        for (int e = t; e < 2 * kHeadDim; e += kThreads / 2)
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

    // 16-byte chunk of a head: dims dv .. dv+7 (values; keys in plain mode);
    // fused keys take the prologue's dims d1 .. d1+3 and d1+16 .. d1+19
    const int dv = 8 * (t & 7);
    const int d1 = prologue::lane_dim(lane);
    const bool split_keys = kFused && keys;
    const int o1 = 2 * (split_keys ? d1 : dv), o2 = 2 * (split_keys ? d1 + 16 : dv + 4);
    const uint8_t* in = reinterpret_cast<const uint8_t*>(keys ? job.k : job.v);
    float sv[4], cv[4];

    for (int h0 = 0; h0 < job.H; h0 += kThreads / 16) {
        const int h = h0 + (t >> 3);
        const bool live = h < job.H;
        uint64_t acc[4] = {0, 0, 0, 0};
        uint2 c_lo = make_uint2(0, 0), c_hi = make_uint2(0, 0);  // a copied token's values
        if (live) {
            const size_t hoff = static_cast<size_t>(h) * kHeadDim * 2;
            if (src.copy) {
                const uint8_t* p = in + (src0 + src.first) * tok_b + hoff;
                c_lo = __ldg(reinterpret_cast<const uint2*>(p + o1));
                c_hi = __ldg(reinterpret_cast<const uint2*>(p + o2));
            } else {
                const uint8_t* p = in + (grid0 + static_cast<size_t>(src.r0) * L.grid_w + src.c0) * tok_b + hoff;
                const size_t row_skip = static_cast<size_t>(L.grid_w - cw) * tok_b;
                int c = 0;
                for (int m0 = 0; m0 < n; m0 += kBatch) {
                    uint2 lo[kBatch], hi[kBatch];
#pragma unroll
                    for (int j = 0; j < kBatch; ++j) {
                        if (m0 + j < n) {
                            lo[j] = __ldg(reinterpret_cast<const uint2*>(p + o1));
                            hi[j] = __ldg(reinterpret_cast<const uint2*>(p + o2));
                            p += tok_b;
                            if (++c == cw) {
                                c = 0;
                                p += row_skip;
                            }
                        }
                    }
#pragma unroll
                    for (int j = 0; j < kBatch; ++j)
                        if (m0 + j < n) add8x2(acc, lo[j], hi[j]);
                }
                if (pow2) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[e] = f2_mul(acc[e], inv2);
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float x, y;
                        f2_unpack(acc[e], x, y);
                        acc[e] = f2_pack(__fdiv_rn(x, count), __fdiv_rn(y, count));
                    }
                }
            }
            if (!split_keys) {  // the means (or the copied token), bf16, token-major
                uint4 o;
                if (src.copy) {
                    o = make_uint4(c_lo.x, c_lo.y, c_hi.x, c_hi.y);
                } else {
                    float m[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) f2_unpack(acc[e], m[2 * e], m[2 * e + 1]);
                    o = make_uint4(prologue::pack2(m[0], m[1]), prologue::pack2(m[2], m[3]),
                                   prologue::pack2(m[4], m[5]), prologue::pack2(m[6], m[7]));
                }
                uint16_t* out = (keys ? job.k_out : job.v_out) + dst * tok + static_cast<size_t>(h) * kHeadDim + dv;
                *reinterpret_cast<uint4*>(out) = o;
            }
        }
        if (!split_keys) continue;  // warp-uniform
        if (h0 == 0) {
            named_bar_sync(kKeyBar, kKeyBarThreads);  // pooled_pos and the staged affine
            prologue::token_angles(pooled_pos, lane, prologue::lane_freq(freq, lane), sv, cv);
        }
        // the pooled keys as stored (bf16; precise mode: the fp32 means), then
        // the prologue
        float x1[4], x2[4];
        if (src.copy) {
            x1[0] = prologue::bf16_lo(c_lo.x); x1[1] = prologue::bf16_hi(c_lo.x);
            x1[2] = prologue::bf16_lo(c_lo.y); x1[3] = prologue::bf16_hi(c_lo.y);
            x2[0] = prologue::bf16_lo(c_hi.x); x2[1] = prologue::bf16_hi(c_hi.x);
            x2[2] = prologue::bf16_lo(c_hi.y); x2[3] = prologue::bf16_hi(c_hi.y);
        } else {
            float m[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) f2_unpack(acc[e], m[2 * e], m[2 * e + 1]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x1[e] = kPrecise ? m[e] : __bfloat162float(__float2bfloat16_rn(m[e]));
                x2[e] = kPrecise ? m[4 + e] : __bfloat162float(__float2bfloat16_rn(m[4 + e]));
            }
        }
        const size_t orow = (static_cast<size_t>(h) * job.k_hat_stride + dst) * kHeadDim;
        if constexpr (kPrecise) {
            float r1[4], r2[4];
            prologue::norm_rotate<kAffine>(x1, x2, aff, sv, cv, d1, r1, r2);
            if (live) prologue::store_two_terms(job.k_hat + orow, job.k_hat_lo + orow, d1, r1, r2);
        } else {
            prologue::norm_rotate_store<kAffine>(x1, x2, aff, sv, cv, live, job.k_hat + orow, d1);
        }
    }
}

template <bool kFused, bool kAffine, bool kPrecise = false>
cudaError_t launch_pool_kernel(const PoolJob& job, unsigned blocks, cudaStream_t stream) {
    kv_pool_kernel<kFused, kAffine, kPrecise><<<blocks, kThreads, 0, stream>>>(job, rope_freq_table());
    return cudaPeekAtLastError();
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
