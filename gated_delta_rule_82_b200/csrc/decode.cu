// decode.cu -- single-token CKDA step over a caller-owned fp32 state, in place.
//
// Per (sequence n, head h), with q, k prepared (rotation at pos[n], then L2 norm):
//     S' = Diag(alpha) S,   w = S'^T k,   y = S'^T q
//     S  <- S' + beta k (v - w)^T                 = (I - beta k k^T) Diag(alpha) S + beta k v^T
//     o   = scale * S^T q = scale * (y + beta (k.q) (v - w))
// (transition of the "Complex KDA" paper summary, "Background"; read-out o_t = dk^-1/2 S_t^T q_t).
//
// The step is HBM-bound: 2 * dk * dv * 4 bytes of state per head against ~7 dk dv flops.  Each
// thread owns a 4-column strip of R rows of one head's state and keeps it in registers between
// the read and the write, so the state crosses HBM exactly once in each direction.  All state
// loads are issued before anything else (128-bit, streaming / evict-first, since a 64 KiB head
// state is never reused within a step); the column reductions w and y go through shared memory;
// the write-back is a 128-bit streaming store.
#include "internal.cuh"

namespace ckda {

namespace {

constexpr int kDecodeThreads = 256;

template <int DK, int DV>
struct DecodeShape {
    static constexpr int C4 = DV / 4;              // threads across a row (float4 each)
    static constexpr int R = DK < 16 ? DK : 16;    // rows per thread
    static constexpr int RG = DK / R;              // row groups
    static constexpr int TPH = C4 * RG;            // threads per head
    static constexpr int HPC = kDecodeThreads / TPH;  // heads per CTA
    static_assert(TPH <= kDecodeThreads && kDecodeThreads % TPH == 0, "bad decode shape");
};

__device__ __forceinline__ float4 ld_stream(const float* p) {
    float4 v;
    asm volatile("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ void st_stream(float* p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}

// Loads of the small per-head vectors, as volatile asm so that they keep their place ahead of the
// state loads: issued first, they return long before the 64 KiB of state behind them, and the
// q/k preparation overlaps the state's arrival.
__device__ __forceinline__ float ld_vec(const float* p) {
    float x;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(x) : "l"(p));
    return x;
}
__device__ __forceinline__ float ld_vec(const __nv_bfloat16* p) {
    unsigned short x;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(x) : "l"(p));
    return __bfloat162float(__ushort_as_bfloat16(x));
}

// kRope: the rotation is compiled in only where it is asked for (the step is latency-bound per CTA
// at two CTAs per SM, so code that a call does not need is left out of its kernel).
template <typename T, int DK, int DV, bool kLogits, bool kRope>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
              const void* __restrict__ alpha, const float* __restrict__ beta,
              float* __restrict__ state, T* __restrict__ out, const long long* __restrict__ pos,
              int NH, int H, int G, int l2norm, RopeParams rp, float scale) {
    using S = DecodeShape<DK, DV>;
    constexpr int HPC = S::HPC, TPH = S::TPH, R = S::R, RG = S::RG, C4 = S::C4;

    __shared__ float sq[HPC][DK], sk[HPC][DK], sa[HPC][DK], sv[HPC][DV];
    __shared__ float sbeta[HPC], skq[HPC];
    __shared__ unsigned long long sfreq[DK / 2];   // RoPE frequencies (lanes index them per channel)
    __shared__ float4 red_w[HPC][RG][C4], red_y[HPC][RG][C4];

    const int tid = threadIdx.x;
    const int hl = tid / TPH, th = tid % TPH;
    const int c4 = th % C4, rg = th / C4;
    const int head = blockIdx.x * HPC + hl;
    const bool valid = head < NH;

    // 1. the per-head vectors (q, k, alpha: NQ elements a thread, v: NV) are requested first
    constexpr int NQ = (HPC * DK + kDecodeThreads - 1) / kDecodeThreads;
    constexpr int NV = (HPC * DV + kDecodeThreads - 1) / kDecodeThreads;
    float qv[NQ], kv[NQ], av[NQ], vv[NV], bv = 0.f;
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        const int e = tid + i * kDecodeThreads, hh = e / DK, c = e % DK;
        const int g = blockIdx.x * HPC + hh;
        qv[i] = kv[i] = av[i] = 0.f;
        if (e < HPC * DK && g < NH) {
            // value head g reads q/k head g / G (grouped value heads; G = 1 without grouping)
            const int gq = G == 1 ? g : g / G;
            qv[i] = ld_vec(q + (size_t)gq * DK + c);
            kv[i] = ld_vec(k + (size_t)gq * DK + c);
            // gate values (fp32), or logits a in the activation type (alpha = 2 sigma(a) - 1 below)
            if constexpr (kLogits)
                av[i] = ld_vec(static_cast<const T*>(alpha) + (size_t)g * DK + c);
            else
                av[i] = ld_vec(static_cast<const float*>(alpha) + (size_t)g * DK + c);
        }
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = tid + i * kDecodeThreads, hh = e / DV, c = e % DV;
        const int g = blockIdx.x * HPC + hh;
        vv[i] = (e < HPC * DV && g < NH) ? ld_vec(v + (size_t)g * DV + c) : 0.f;
    }
    if (tid < HPC && blockIdx.x * HPC + tid < NH) bv = ld_vec(beta + blockIdx.x * HPC + tid);

    // 2. then this thread's strip of the state (consumed last)
    float4 s[R];
    float* sbase = state + (size_t)(valid ? head : 0) * DK * DV + c4 * 4;
    if (valid) {
#pragma unroll
        for (int j = 0; j < R; ++j) s[j] = ld_stream(sbase + (size_t)(rg + j * RG) * DV);
    }

    // 3. the vectors into shared memory (fp32)
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        const int e = tid + i * kDecodeThreads;
        if (e < HPC * DK) {
            sq[e / DK][e % DK] = qv[i];
            sk[e / DK][e % DK] = kv[i];
            sa[e / DK][e % DK] = kLogits ? gate_alpha(av[i]) : av[i];
        }
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = tid + i * kDecodeThreads;
        if (e < HPC * DV) sv[e / DV][e % DV] = vv[i];
    }
    if (kRope)
        for (int i = tid; i < DK / 2; i += kDecodeThreads) sfreq[i] = rp.turns[i];
    if (tid < HPC) sbeta[tid] = (kLogits && blockIdx.x * HPC + tid < NH) ? gate_beta(bv) : bv;
    __syncthreads();

    // 4. rotation and L2 norm of q and k: one warp per head
    const int lane = tid & 31, warp = tid >> 5;
    for (int hh = warp; hh < HPC; hh += kDecodeThreads / 32) {
        int g = blockIdx.x * HPC + hh;
        constexpr int PER = (DK + 31) / 32;
        float qr[PER], kr[PER];
#pragma unroll
        for (int m = 0; m < PER; ++m) {
            int c = lane + 32 * m;
            qr[m] = c < DK ? sq[hh][c] : 0.f;
            kr[m] = c < DK ? sk[hh][c] : 0.f;
        }
        if (kRope && g < NH) {
            long long p = pos[g / H];
#pragma unroll
            for (int m = 0; m < PER; ++m) {
                int c = lane + 32 * m;
                if (c < rp.rot_dims) {   // the first rot_dims channels rotate
                    int i, partner;
                    bool first;
                    if (rp.convention == 0) {
                        const int half = rp.rot_dims / 2;
                        i = c % half; first = c < half; partner = first ? c + half : c - half;
                    } else {
                        i = c / 2; first = (c & 1) == 0; partner = c ^ 1;
                    }
                    float sn, cs;
                    rope_sincos(p, sfreq[i], &sn, &cs);
                    float qp = sq[hh][partner], kp = sk[hh][partner];
                    qr[m] = first ? qr[m] * cs - qp * sn : qr[m] * cs + qp * sn;
                    kr[m] = first ? kr[m] * cs - kp * sn : kr[m] * cs + kp * sn;
                }
            }
        }
        if (l2norm) {
            float ssq = 0.f, ssk = 0.f;
#pragma unroll
            for (int m = 0; m < PER; ++m) { ssq += qr[m] * qr[m]; ssk += kr[m] * kr[m]; }
            ssq = warp_sum(ssq);
            ssk = warp_sum(ssk);
            float rq = rsqrtf(ssq + kL2Eps), rk = rsqrtf(ssk + kL2Eps);
#pragma unroll
            for (int m = 0; m < PER; ++m) { qr[m] *= rq; kr[m] *= rk; }
        }
        float dot = 0.f;
#pragma unroll
        for (int m = 0; m < PER; ++m) dot += qr[m] * kr[m];
        dot = warp_sum(dot);
        __syncwarp();
#pragma unroll
        for (int m = 0; m < PER; ++m) {
            int c = lane + 32 * m;
            if (c < DK) { sq[hh][c] = qr[m]; sk[hh][c] = kr[m]; }
        }
        if (lane == 0) skq[hh] = dot;
    }
    __syncthreads();

    // 5. gate the rows and reduce w = S'^T k, y = S'^T q over this thread's rows
    float4 w = make_float4(0.f, 0.f, 0.f, 0.f), y = w;
    if (valid) {
#pragma unroll
        for (int j = 0; j < R; ++j) {
            int c = rg + j * RG;
            float a = sa[hl][c], kc = sk[hl][c], qc = sq[hl][c];
            s[j].x *= a; s[j].y *= a; s[j].z *= a; s[j].w *= a;
            w.x += s[j].x * kc; w.y += s[j].y * kc; w.z += s[j].z * kc; w.w += s[j].w * kc;
            y.x += s[j].x * qc; y.y += s[j].y * qc; y.z += s[j].z * qc; y.w += s[j].w * qc;
        }
    }
    red_w[hl][rg][c4] = w;
    red_y[hl][rg][c4] = y;
    __syncthreads();
    w = make_float4(0.f, 0.f, 0.f, 0.f);
    y = w;
#pragma unroll
    for (int g2 = 0; g2 < RG; ++g2) {
        float4 a = red_w[hl][g2][c4], b = red_y[hl][g2][c4];
        w.x += a.x; w.y += a.y; w.z += a.z; w.w += a.w;
        y.x += b.x; y.y += b.y; y.z += b.z; y.w += b.w;
    }
    if (!valid) return;

    // 6. rank-one write and read-out
    const float bt = sbeta[hl];
    float4 u;
    u.x = bt * (sv[hl][c4 * 4 + 0] - w.x);
    u.y = bt * (sv[hl][c4 * 4 + 1] - w.y);
    u.z = bt * (sv[hl][c4 * 4 + 2] - w.z);
    u.w = bt * (sv[hl][c4 * 4 + 3] - w.w);
#pragma unroll
    for (int j = 0; j < R; ++j) {
        int c = rg + j * RG;
        float kc = sk[hl][c];
        float4 r = s[j];
        r.x += kc * u.x; r.y += kc * u.y; r.z += kc * u.z; r.w += kc * u.w;
        st_stream(sbase + (size_t)c * DV, r);
    }
    if (rg == 0) {
        float kq = skq[hl];
        T* o = out + (size_t)head * DV + c4 * 4;
        o[0] = from_f32<T>(scale * (y.x + kq * u.x));
        o[1] = from_f32<T>(scale * (y.y + kq * u.y));
        o[2] = from_f32<T>(scale * (y.z + kq * u.z));
        o[3] = from_f32<T>(scale * (y.w + kq * u.w));
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const void* alpha,
                            const float* beta, float* state, void* out, const long long* pos,
                            int N, int H, int G, int l2norm, const RopeParams& rp, float scale,
                            int gate_logits, cudaStream_t stream) {
    using S = DecodeShape<DK, DV>;
    int NH = N * H;
    int grid = (NH + S::HPC - 1) / S::HPC;
    auto kern = gate_logits ? (rp.enabled ? decode_kernel<T, DK, DV, true, true>
                                          : decode_kernel<T, DK, DV, true, false>)
                            : (rp.enabled ? decode_kernel<T, DK, DV, false, true>
                                          : decode_kernel<T, DK, DV, false, false>);
    kern<<<grid, kDecodeThreads, 0, stream>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), alpha, beta,
        state, static_cast<T*>(out), pos, NH, H, G, l2norm, rp, scale);
    return cudaGetLastError();
}

template <typename T, int DK>
cudaError_t dispatch_dv(int dv, const void* q, const void* k, const void* v, const void* alpha,
                        const float* beta, float* state, void* out, const long long* pos, int N,
                        int H, int G, int l2norm, const RopeParams& rp, float scale,
                        int gate_logits, cudaStream_t stream) {
    switch (dv) {
        case 16: return launch_decode_t<T, DK, 16>(q, k, v, alpha, beta, state, out, pos, N, H, G, l2norm, rp, scale, gate_logits, stream);
        case 32: return launch_decode_t<T, DK, 32>(q, k, v, alpha, beta, state, out, pos, N, H, G, l2norm, rp, scale, gate_logits, stream);
        case 64: return launch_decode_t<T, DK, 64>(q, k, v, alpha, beta, state, out, pos, N, H, G, l2norm, rp, scale, gate_logits, stream);
        case 128: return launch_decode_t<T, DK, 128>(q, k, v, alpha, beta, state, out, pos, N, H, G, l2norm, rp, scale, gate_logits, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t dispatch_dk(int dk, int dv, const void* q, const void* k, const void* v,
                        const void* alpha, const float* beta, float* state, void* out,
                        const long long* pos, int N, int H, int G, int l2norm, const RopeParams& rp,
                        float scale, int gate_logits, cudaStream_t stream) {
    switch (dk) {
        case 16: return dispatch_dv<T, 16>(dv, q, k, v, alpha, beta, state, out, pos, N, H, G, l2norm, rp, scale, gate_logits, stream);
        case 32: return dispatch_dv<T, 32>(dv, q, k, v, alpha, beta, state, out, pos, N, H, G, l2norm, rp, scale, gate_logits, stream);
        case 64: return dispatch_dv<T, 64>(dv, q, k, v, alpha, beta, state, out, pos, N, H, G, l2norm, rp, scale, gate_logits, stream);
        case 128: return dispatch_dv<T, 128>(dv, q, k, v, alpha, beta, state, out, pos, N, H, G, l2norm, rp, scale, gate_logits, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* alpha,
                          const float* beta, float* state, void* out, const long long* pos, int N,
                          int H, int G, int dk, int dv, int l2norm, const RopeParams& rp, float scale,
                          int gate_logits, ckda_dtype dtype, cudaStream_t stream) {
    if (dtype == CKDA_BF16)
        return dispatch_dk<__nv_bfloat16>(dk, dv, q, k, v, alpha, beta, state, out, pos, N, H, G,
                                          l2norm, rp, scale, gate_logits, stream);
    return dispatch_dk<float>(dk, dv, q, k, v, alpha, beta, state, out, pos, N, H, G, l2norm, rp,
                              scale, gate_logits, stream);
}

}  // namespace ckda
