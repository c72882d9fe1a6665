// prologue.cu -- q/k prologue: rotary embedding, then the per-head L2 norm.
//
// The rotation pairs (x_i, x_{i+dk/2}) (rotate_half) or (x_{2i}, x_{2i+1}) (interleaved) and
// turns each pair by (pos_offset + t) * theta^(-2i/dk); the L2 norm x / sqrt(sum x^2 + 1e-6)
// follows it ("RoPE into the KDA q/k path" review, sections 2, 3 and 5).
//
// Layout: one CTA handles a run of consecutive tokens (all their heads, q and k).  Each head
// vector is held by a group of G lanes with 16-byte loads and stores (8 bf16 or 4 fp32 per lane),
// and the norm is a G-lane shuffle reduction.  Every thread first issues the loads of all its
// vectors (up to kMaxRounds per batch, kept as raw 16-byte words), so that many bytes are in
// flight per SM; the sin/cos of the run's angles are computed into shared memory while they
// arrive, shared by the 2*H head vectors of each token.  The kernel reads and writes every q/k
// element once: it is HBM-bound.
#include "internal.cuh"

namespace ckda {

namespace {

constexpr int kPrologueThreads = 256;
constexpr int kMaxRounds = 8;      // head vectors per thread per batch
constexpr int kMaxTokPerCta = 64;  // bounds the sin/cos table (64 x 64 float2 = 32 KB)

// vectors of one CTA round (all warps)
template <typename T, int DK>
constexpr int vectors_per_round() {
    return (kPrologueThreads / 32) * (32 / (DK / ElemsPer16<T>::value));
}

template <typename T, int DK>
__global__ void __launch_bounds__(kPrologueThreads)
qk_prologue_kernel(const T* __restrict__ q, const T* __restrict__ k, T* __restrict__ qo,
                   T* __restrict__ ko, int BT, int T_len, int H, int tok_per_cta, int l2norm,
                   RopeParams rp, long long pos_offset) {
    constexpr int EPL = ElemsPer16<T>::value;  // elements per lane
    constexpr int G = DK / EPL;                // lanes per head vector
    constexpr int VPW = 32 / G;                // head vectors per warp instruction
    constexpr int VPR = vectors_per_round<T, DK>();
    constexpr int HALF = DK / 2;
    static_assert(G >= 2 && G <= 32, "unsupported head size for this element type");

    extern __shared__ float2 cs[];   // (cos, sin) [token of the run][frequency]
    __shared__ double sfreq[HALF];

    const int tok0 = blockIdx.x * tok_per_cta;
    const int ntok = min(tok_per_cta, BT - tok0);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / G, li = lane % G;
    const int nvec = ntok * 2 * H;  // (token, q/k, head)
    const int two_h = 2 * H;
    for (int b0 = 0; b0 < nvec; b0 += kMaxRounds * VPR) {
        // 1. issue every load of this batch (vector b0 + r VPR + warp VPW + grp in round r)
        uint4 raw[kMaxRounds];
#pragma unroll
        for (int r = 0; r < kMaxRounds; ++r) {
            const int vid = b0 + r * VPR + warp * VPW + grp;
            if (vid < nvec) {
                const int j = vid / two_h, rem = vid - j * two_h;
                const int which = rem >= H, h = which ? rem - H : rem;
                const T* src = which ? k : q;
                raw[r] = __ldcs(reinterpret_cast<const uint4*>(
                    src + ((size_t)(tok0 + j) * H + h) * DK + (size_t)li * EPL));
            }
        }
        // 2. the run's sin/cos table, once, while the loads are in flight
        if (rp.enabled && b0 == 0) {
            for (int i = threadIdx.x; i < HALF; i += blockDim.x) sfreq[i] = rp.inv_freq[i];
            __syncthreads();
            for (int e = threadIdx.x; e < ntok * HALF; e += blockDim.x) {
                const int j = e / HALF, i = e - j * HALF;
                const int t = (tok0 + j) % T_len;
                float sn, c;
                rope_sincos(pos_offset + t, sfreq[i], &sn, &c);
                cs[j * HALF + i] = make_float2(c, sn);
            }
            __syncthreads();
        }
        // 3. rotate, normalise, store
#pragma unroll
        for (int r = 0; r < kMaxRounds; ++r) {
            const int vid = b0 + r * VPR + warp * VPW + grp;
            if (b0 + r * VPR >= nvec) break;   // warp-uniform: no later round has a vector
            const bool active = vid < nvec;
            const int vv = active ? vid : 0;
            const int j = vv / two_h, rem = vv - j * two_h;
            const int which = rem >= H, h = which ? rem - H : rem;
            float x[EPL];
            if (active) {
                if constexpr (EPL == 8) {
                    const uint32_t w[4] = {raw[r].x, raw[r].y, raw[r].z, raw[r].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        x[2 * e] = __uint_as_float(w[e] << 16);
                        x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                    }
                } else {
                    x[0] = __uint_as_float(raw[r].x); x[1] = __uint_as_float(raw[r].y);
                    x[2] = __uint_as_float(raw[r].z); x[3] = __uint_as_float(raw[r].w);
                }
            } else {
#pragma unroll
                for (int e = 0; e < EPL; ++e) x[e] = 0.f;
            }
            if (rp.enabled) {
                // the first rot_dims channels rotate (all of them, or the first half of the head)
                const int rot = rp.rot_dims;
                const float2* csj = cs + j * HALF;
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
                            const int i = (li * EPL + e) % (rot / 2);
                            const float2 c = csj[i];
                            x[e] = first ? (x[e] * c.x - y[e] * c.y) : (x[e] * c.x + y[e] * c.y);
                        }
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < EPL; e += 2) {
                        if (li * EPL + e >= rot) continue;
                        const float2 c = csj[(li * EPL + e) / 2];
                        const float a = x[e], b = x[e + 1];
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
                const float rn = rsqrtf(ss + kL2Eps);
#pragma unroll
                for (int e = 0; e < EPL; ++e) x[e] *= rn;
            }
            if (active) {
                T* dst = which ? ko : qo;
                Vec16<T, EPL>::store(dst + ((size_t)(tok0 + j) * H + h) * DK + (size_t)li * EPL, x);
            }
        }
    }
}

template <typename T, int DK>
cudaError_t launch_prologue_t(const void* q, const void* k, void* qo, void* ko, int B, int T_len,
                              int H, int l2norm, const RopeParams& rp, long long pos_offset,
                              cudaStream_t stream) {
    const int BT = B * T_len;
    // tokens per CTA: one batch of kMaxRounds vectors per thread covers them (at least one
    // token, at most kMaxTokPerCta)
    constexpr int per_batch = kMaxRounds * vectors_per_round<T, DK>();
    const int tpc = max(1, min(kMaxTokPerCta, per_batch / (2 * H)));
    const int grid = (BT + tpc - 1) / tpc;
    const size_t smem = rp.enabled ? (size_t)tpc * (DK / 2) * sizeof(float2) : 0;
    qk_prologue_kernel<T, DK><<<grid, kPrologueThreads, smem, stream>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<T*>(qo),
        static_cast<T*>(ko), BT, T_len, H, tpc, l2norm, rp, pos_offset);
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
