// simt_chunk.cuh -- the per-chunk factors of the chunked CKDA recurrence on CUDA cores (fp32),
// shared by the SIMT forward (chunk_simt.cu) and the backward (chunk_bwd.cu).
//
// For a chunk of C tokens r = 0..C-1 (derived from the transition of the "Complex KDA" paper
// summary, "Background": A_t = (I - beta_t k_t k_t^T) Diag(alpha_t)):
//   q^, k^   the prepared rows (rotation, then L2 norm; "RoPE review", sections 2-3)
//   sigma_r  the running sign product of the gates per channel, absorbed into q' = sigma q^ and
//            k' = sigma k^ (the sign-magnitude split of the summary's Proposition 2)
//   L_r      the running sum of log2 |alpha| per channel (|alpha| floored at FLT_MIN), so that
//            every ratio |gamma_r| / |gamma_j| (j <= r) is exp2(L_r - L_j) <= 1
//   A_rj = beta_r k'_r . R_rj k'_j (j < r),  M_rj = q'_r . R_rj k'_j (j <= r),  R_rj = exp2(L_r - L_j)
//   T = (I + A)^-1,  W = T diag(beta) K_gamma  (K_gamma,r = exp2(L_r) k'_r)
// Rows past the valid length are identity steps (alpha = 1, beta = 0, q = k = v = 0).
#pragma once

#include "internal.cuh"

namespace ckda {
namespace simt {

constexpr int kThreads = 256;   // >= 128 (one thread per channel) and >= the chunk
constexpr float kFltMin = 1.17549435e-38f;

// Shared-memory arrays of one chunk's factors (floats).  The rows of q', k', L and W are LD =
// DK + 1 floats apart, so that loops whose lanes run over rows at a fixed channel (the A and M
// products) hit distinct banks.
template <int DK, int C>
struct Factors {
    static constexpr int LD = DK + 1;
    float* q;    // q'  [C][LD]
    float* k;    // k'  [C][LD]
    float* L;    // L   [C][LD]
    float* W;    // W   [C][LD]
    float* A;    // A   [C][C]
    float* M;    // M   [C][C]
    float* T;    // T   [C][C]
    float* b;    // beta [C]
    float* sg;   // sigma_C [DK]
    float* LC;   // L_C [DK]
    static constexpr int floats = 4 * C * LD + 3 * C * C + C + 2 * DK;
    __device__ void bind(float* p) {
        q = p; k = q + C * LD; L = k + C * LD; W = L + C * LD; A = W + C * LD; M = A + C * C;
        T = M + C * C; b = T + C * C; sg = b + C; LC = sg + DK;
    }
    // without W and A (for a kernel that takes M and T from elsewhere)
    static constexpr int floats_nw = 3 * C * LD + 2 * C * C + C + 2 * DK;
    __device__ void bind_nw(float* p) {
        q = p; k = q + C * LD; L = k + C * LD; W = nullptr; A = nullptr; M = L + C * LD;
        T = M + C * C; b = T + C * C; sg = b + C; LC = sg + DK;
    }
};

// Rows r < nvalid of q and k (value head h reads q/k row (token * H + h) / G), beta of head h,
// alpha from fp32 values or `dtype` logits; rows past nvalid are identity steps.  Then the
// prologue (rotation at position pos0 + r, L2 norm) and the gate prefix with the signs absorbed:
// q', k', L, beta, sigma_C and L_C.  `first` is the token index of row 0 on the token axis.
// alpha_out (nullable, [C][DK]) receives the gates themselves (1 past nvalid).  Ends with a
// barrier.
template <typename Tin, int DK, int C>
__device__ __forceinline__ void chunk_prep(const Factors<DK, C>& f, const Tin* __restrict__ q,
                                              const Tin* __restrict__ k,
                                              const void* __restrict__ alpha,
                                              const float* __restrict__ beta, size_t first, int t0,
                                              int nvalid, int H, int h, int G, int l2norm,
                                              const RopeParams& rp, const unsigned long long* sfreq,
                                              long long pos0, int gate_logits,
                                              float* alpha_out = nullptr) {
    constexpr int LD = Factors<DK, C>::LD;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kThreads / 32;
    // the chunk's global loads are issued in batches before their values are used: q and k in
    // groups of up to 8 elements per thread, beta, and the gates of this thread's channel
    // (thread c < DK) for the first rows (the later rows are loaded, again in batches, during
    // the gate prefix below)
    constexpr int NQK = (C * DK + kThreads - 1) / kThreads;
    constexpr int QG = NQK < 8 ? NQK : 8;
    constexpr int AG = C < 16 ? C : 16;
    auto gate_at = [&](int r) {
        const size_t ia = ((first + t0 + r) * H + h) * DK + tid;
        return r >= nvalid ? 1.f
               : gate_logits ? gate_alpha(to_f32(static_cast<const Tin*>(alpha)[ia]))
                             : static_cast<const float*>(alpha)[ia];
    };
    float av[AG];
    float bv = tid < nvalid ? beta[(first + t0 + tid) * H + h] : 0.f;
    if (tid < DK) {
#pragma unroll
        for (int r = 0; r < AG; ++r) av[r] = gate_at(r);
    }
    for (int i0 = 0; i0 < NQK; i0 += QG) {
        float qv[QG], kv[QG];
#pragma unroll
        for (int i = 0; i < QG; ++i) {
            const int e = tid + (i0 + i) * kThreads, r = e / DK, c = e % DK;
            qv[i] = kv[i] = 0.f;
            if (e < C * DK && r < nvalid) {
                const size_t row = ((first + t0 + r) * H + h) / G;
                qv[i] = to_f32(q[row * DK + c]);
                kv[i] = to_f32(k[row * DK + c]);
            }
        }
#pragma unroll
        for (int i = 0; i < QG; ++i) {
            const int e = tid + (i0 + i) * kThreads, r = e / DK, c = e % DK;
            if (e < C * DK) {
                f.q[r * LD + c] = qv[i];
                f.k[r * LD + c] = kv[i];
            }
        }
    }
    if (tid < C) {
        if (tid < nvalid && gate_logits) bv = gate_beta(bv);   // beta = 2 sigma(b)
        f.b[tid] = bv;
    }
    __syncthreads();
    // prologue per row (one warp per row): rotation, then L2 norm
    for (int r = warp; r < nvalid; r += NW) {
        constexpr int PER = (DK + 31) / 32;
        float qr[PER], kr[PER];
        const long long p = pos0 + r;
#pragma unroll
        for (int m = 0; m < PER; ++m) {
            const int c = lane + 32 * m;
            qr[m] = c < DK ? f.q[r * LD + c] : 0.f;
            kr[m] = c < DK ? f.k[r * LD + c] : 0.f;
            if (rp.enabled && c < rp.rot_dims) {   // the first rot_dims channels rotate
                int i, partner;
                bool lo;
                if (rp.convention == 0) {
                    const int half = rp.rot_dims / 2;
                    i = c % half; lo = c < half; partner = lo ? c + half : c - half;
                } else {
                    i = c / 2; lo = (c & 1) == 0; partner = c ^ 1;
                }
                float sn, cs;
                rope_sincos(p, sfreq[i], &sn, &cs);
                const float qp = f.q[r * LD + partner], kp = f.k[r * LD + partner];
                qr[m] = lo ? qr[m] * cs - qp * sn : qr[m] * cs + qp * sn;
                kr[m] = lo ? kr[m] * cs - kp * sn : kr[m] * cs + kp * sn;
            }
        }
        if (l2norm) {
            float a = 0.f, bb = 0.f;
#pragma unroll
            for (int m = 0; m < PER; ++m) { a += qr[m] * qr[m]; bb += kr[m] * kr[m]; }
            a = rsqrtf(warp_sum(a) + kL2Eps);
            bb = rsqrtf(warp_sum(bb) + kL2Eps);
#pragma unroll
            for (int m = 0; m < PER; ++m) { qr[m] *= a; kr[m] *= bb; }
        }
        __syncwarp();
#pragma unroll
        for (int m = 0; m < PER; ++m) {
            const int c = lane + 32 * m;
            if (c < DK) { f.q[r * LD + c] = qr[m]; f.k[r * LD + c] = kr[m]; }
        }
    }
    __syncthreads();
    // gate prep: sign parity and log2-magnitude prefix per channel; absorb signs
    if (tid < DK) {
        const int c = tid;
        float L = 0.f, sg = 1.f;
#pragma unroll
        for (int r0 = 0; r0 < C; r0 += AG) {
            if (r0 > 0) {
#pragma unroll
                for (int r = 0; r < AG; ++r) av[r] = gate_at(r0 + r);
            }
#pragma unroll
            for (int r = 0; r < AG; ++r) {
                const float a = av[r];
                if (alpha_out) alpha_out[(r0 + r) * DK + c] = a;
                if (a < 0.f) sg = -sg;
                L += log2f(fmaxf(fabsf(a), kFltMin));
                f.L[(r0 + r) * LD + c] = L;
                f.q[(r0 + r) * LD + c] *= sg;
                f.k[(r0 + r) * LD + c] *= sg;
            }
        }
        f.sg[c] = sg;
        f.LC[c] = L;
    }
    __syncthreads();
}

// A, M, T and W of a chunk whose q', k', L and beta chunk_prep has filled in; P (nullable, [C][C])
// receives A before the row scaling by beta.  Ends with a barrier.
template <int DK, int C>
__device__ __forceinline__ void chunk_products(const Factors<DK, C>& f, float* P = nullptr) {
    constexpr int LD = Factors<DK, C>::LD;
    const int tid = threadIdx.x;
    // A (strictly lower) and M (lower incl. diagonal)
    for (int e = tid; e < C * C; e += kThreads) {
        const int r = e / C, j = e % C;
        float a = 0.f, m = 0.f;
        if (j <= r) {
            for (int c = 0; c < DK; ++c) {
                const float kk = f.k[j * LD + c] * exp2f(f.L[r * LD + c] - f.L[j * LD + c]);
                a += f.k[r * LD + c] * kk;
                m += f.q[r * LD + c] * kk;
            }
            if (j == r) a = 0.f;
        }
        if (P) P[e] = a;
        f.A[e] = a * f.b[r];
        f.M[e] = m;
    }
    __syncthreads();
    // T = (I + A)^-1 by forward substitution, one column per thread
    for (int j = tid; j < C; j += kThreads) {
        for (int r = 0; r < C; ++r) {
            float t;
            if (r < j) t = 0.f;
            else if (r == j) t = 1.f;
            else {
                float acc = 0.f;
                for (int m = j; m < r; ++m) acc += f.A[r * C + m] * f.T[m * C + j];
                t = -acc;
            }
            f.T[r * C + j] = t;
        }
    }
    __syncthreads();
    // W = T diag(beta) K_gamma
    for (int e = tid; e < C * DK; e += kThreads) {
        const int r = e / DK, c = e % DK;
        float acc = 0.f;
        for (int j = 0; j <= r; ++j)
            acc += f.T[r * C + j] * f.b[j] * exp2f(f.L[j * LD + c]) * f.k[j * LD + c];
        f.W[r * LD + c] = acc;
    }
    __syncthreads();
}

// chunk_prep, then chunk_products: every factor of the chunk.
template <typename Tin, int DK, int C>
__device__ __forceinline__ void chunk_factors(const Factors<DK, C>& f, const Tin* __restrict__ q,
                                              const Tin* __restrict__ k,
                                              const void* __restrict__ alpha,
                                              const float* __restrict__ beta, size_t first, int t0,
                                              int nvalid, int H, int h, int G, int l2norm,
                                              const RopeParams& rp, const unsigned long long* sfreq,
                                              long long pos0, int gate_logits) {
    chunk_prep<Tin, DK, C>(f, q, k, alpha, beta, first, t0, nvalid, H, h, G, l2norm, rp, sfreq,
                           pos0, gate_logits);
    chunk_products<DK, C>(f);
}

}  // namespace simt
}  // namespace ckda
