// prologue.cu -- q/k prologue: rotary embedding, then the per-head L2 norm.
//
// The rotation pairs (x_i, x_{i+dk/2}) (rotate_half) or (x_{2i}, x_{2i+1}) (interleaved) and
// turns each pair by (pos_offset + t) * theta^(-2i/dk); the L2 norm x / sqrt(sum x^2 + 1e-6)
// follows it ("RoPE into the KDA q/k path" review, sections 2, 3 and 5).
//
// Layout: one CTA handles kTokPerCta tokens.  The sin/cos of the dk/2 angles of a token are
// computed once into shared memory and shared by the 2*H head vectors of q and k; each head
// vector is held by a group of G lanes with 16-byte loads and stores (8 bf16 or 4 fp32 per lane),
// and the norm is a G-lane shuffle reduction.  The kernel is HBM-bound: it reads and writes
// every q/k element once.
#include "internal.cuh"

namespace ckda {

namespace {

constexpr int kTokPerCta = 4;
constexpr int kPrologueThreads = 256;

template <typename T, int DK>
__global__ void __launch_bounds__(kPrologueThreads)
qk_prologue_kernel(const T* __restrict__ q, const T* __restrict__ k, T* __restrict__ qo,
                   T* __restrict__ ko, int BT, int T_len, int H, int l2norm, RopeParams rp,
                   long long pos_offset) {
    constexpr int EPL = ElemsPer16<T>::value;  // elements per lane
    constexpr int G = DK / EPL;                // lanes per head vector
    constexpr int VPW = 32 / G;                // head vectors per warp instruction
    constexpr int HALF = DK / 2;
    static_assert(G >= 2 && G <= 32, "unsupported head size for this element type");

    __shared__ float2 cs[kTokPerCta][HALF];  // (cos, sin) per token and frequency

    const int tok0 = blockIdx.x * kTokPerCta;
    const int ntok = min(kTokPerCta, BT - tok0);
    if (rp.enabled) {
        // inverse frequencies in shared memory (a per-lane index into the kernel-parameter
        // array would serialise in the constant cache)
        __shared__ double sfreq[HALF];
        for (int i = threadIdx.x; i < HALF; i += blockDim.x) sfreq[i] = rp.inv_freq[i];
        __syncthreads();
        for (int e = threadIdx.x; e < ntok * HALF; e += blockDim.x) {
            int j = e / HALF, i = e % HALF;
            int t = (tok0 + j) % T_len;
            float s, c;
            rope_sincos(pos_offset + t, sfreq[i], &s, &c);
            cs[j][i] = make_float2(c, s);
        }
        __syncthreads();
    }

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / G, li = lane % G;
    const int nvec = ntok * 2 * H;  // (token, q/k, head)
    for (int vbase = warp * VPW; vbase < nvec; vbase += (kPrologueThreads / 32) * VPW) {
        int vid = vbase + grp;
        bool active = vid < nvec;
        int vv = active ? vid : 0;
        int j = vv / (2 * H);
        int rem = vv % (2 * H);
        int which = rem / H, h = rem % H;
        size_t base = ((size_t)(tok0 + j) * H + h) * DK + (size_t)li * EPL;
        const T* src = which ? k : q;
        T* dst = which ? ko : qo;
        float x[EPL];
        if (active) Vec16<T, EPL>::load(src + base, x);
        else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) x[e] = 0.f;
        }
        if (rp.enabled) {
            // the first rot_dims channels rotate (all of them, or the first half of the head)
            const int rot = rp.rot_dims;
            if (rp.convention == 0) {
                // pairs (i, i + rot / 2): the partner's elements are dl lanes away
                const int dl = rot == DK ? G / 2 : G / 4;
                float y[EPL];
#pragma unroll
                for (int e = 0; e < EPL; ++e) y[e] = __shfl_xor_sync(0xffffffffu, x[e], dl);
                const bool first = li < dl;
                if (li < 2 * dl) {
#pragma unroll
                    for (int e = 0; e < EPL; ++e) {
                        int i = (li * EPL + e) % (rot / 2);
                        float2 c = cs[j][i];
                        x[e] = first ? (x[e] * c.x - y[e] * c.y) : (x[e] * c.x + y[e] * c.y);
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < EPL; e += 2) {
                    if (li * EPL + e >= rot) continue;
                    int i = (li * EPL + e) / 2;
                    float2 c = cs[j][i];
                    float a = x[e], b = x[e + 1];
                    x[e] = a * c.x - b * c.y;
                    x[e + 1] = b * c.x + a * c.y;
                }
            }
        }
        if (l2norm) {
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) ss += x[e] * x[e];
            ss = group_sum<G>(ss);
            float r = rsqrtf(ss + kL2Eps);
#pragma unroll
            for (int e = 0; e < EPL; ++e) x[e] *= r;
        }
        if (active) Vec16<T, EPL>::store(dst + base, x);
    }
}

template <typename T, int DK>
cudaError_t launch_prologue_t(const void* q, const void* k, void* qo, void* ko, int B, int T_len,
                              int H, int l2norm, const RopeParams& rp, long long pos_offset,
                              cudaStream_t stream) {
    int BT = B * T_len;
    int grid = (BT + kTokPerCta - 1) / kTokPerCta;
    qk_prologue_kernel<T, DK><<<grid, kPrologueThreads, 0, stream>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<T*>(qo),
        static_cast<T*>(ko), BT, T_len, H, l2norm, rp, pos_offset);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qk_prologue(const void* q, const void* k, void* qo, void* ko, int B, int T_len,
                               int H, int dk, int l2norm, const RopeParams& rp,
                               long long pos_offset, ckda_dtype dtype, cudaStream_t stream) {
#define CKDA_PRO_CASE(TT, D)                                                                  \
    if (dk == D)                                                                             \
        return launch_prologue_t<TT, D>(q, k, qo, ko, B, T_len, H, l2norm, rp, pos_offset, stream);
    if (dtype == CKDA_BF16) {
        CKDA_PRO_CASE(__nv_bfloat16, 16)
        CKDA_PRO_CASE(__nv_bfloat16, 32)
        CKDA_PRO_CASE(__nv_bfloat16, 64)
        CKDA_PRO_CASE(__nv_bfloat16, 128)
    } else {
        CKDA_PRO_CASE(float, 16)
        CKDA_PRO_CASE(float, 32)
        CKDA_PRO_CASE(float, 64)
        CKDA_PRO_CASE(float, 128)
    }
#undef CKDA_PRO_CASE
    return cudaErrorInvalidValue;
}

}  // namespace ckda
