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

constexpr int kThreads = 256;
constexpr float kFltMin = 1.17549435e-38f;

// Shared-memory arrays of one chunk's factors (floats).
template <int DK, int C>
struct Factors {
    float* q;    // q'  [C][DK]
    float* k;    // k'  [C][DK]
    float* L;    // L   [C][DK]
    float* W;    // W   [C][DK]
    float* A;    // A   [C][C]
    float* M;    // M   [C][C]
    float* T;    // T   [C][C]
    float* b;    // beta [C]
    float* sg;   // sigma_C [DK]
    float* LC;   // L_C [DK]
    static constexpr int floats = 4 * C * DK + 3 * C * C + C + 2 * DK;
    __device__ void bind(float* p) {
        q = p; k = q + C * DK; L = k + C * DK; W = L + C * DK; A = W + C * DK; M = A + C * C;
        T = M + C * C; b = T + C * C; sg = b + C; LC = sg + DK;
    }
};

// Rows r < nvalid of q and k (value head h reads q/k row (token * H + h) / G), beta of head h,
// alpha from fp32 values or `dtype` logits; rows past nvalid are identity steps.  Then the
// prologue (rotation at position pos0 + r, L2 norm), the gate prefix with the signs absorbed, A,
// M, T and W.  `first` is the token index of row 0 on the token axis.  Ends with a barrier.
template <typename Tin, int DK, int C>
__device__ __forceinline__ void chunk_factors(const Factors<DK, C>& f, const Tin* __restrict__ q,
                                              const Tin* __restrict__ k,
                                              const void* __restrict__ alpha,
                                              const float* __restrict__ beta, size_t first, int t0,
                                              int nvalid, int H, int h, int G, int l2norm,
                                              const RopeParams& rp, const unsigned long long* sfreq,
                                              long long pos0, int gate_logits) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kThreads / 32;
    for (int e = tid; e < C * DK; e += kThreads) {
        const int r = e / DK, c = e % DK;
        float qv = 0.f, kv = 0.f;
        if (r < nvalid) {
            const size_t row = ((first + t0 + r) * H + h) / G;
            qv = to_f32(q[row * DK + c]);
            kv = to_f32(k[row * DK + c]);
        }
        f.q[e] = qv;
        f.k[e] = kv;
    }
    for (int r = tid; r < C; r += kThreads) {
        float bv = r < nvalid ? beta[(first + t0 + r) * H + h] : 0.f;
        if (r < nvalid && gate_logits) bv = gate_beta(bv);   // beta = 2 sigma(b)
        f.b[r] = bv;
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
            qr[m] = c < DK ? f.q[r * DK + c] : 0.f;
            kr[m] = c < DK ? f.k[r * DK + c] : 0.f;
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
                const float qp = f.q[r * DK + partner], kp = f.k[r * DK + partner];
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
            if (c < DK) { f.q[r * DK + c] = qr[m]; f.k[r * DK + c] = kr[m]; }
        }
    }
    __syncthreads();
    // gate prep: sign parity and log2-magnitude prefix per channel; absorb signs
    for (int c = tid; c < DK; c += kThreads) {
        float L = 0.f, sg = 1.f;
        for (int r = 0; r < C; ++r) {
            float a = 1.f;
            if (r < nvalid) {
                const size_t ia = ((first + t0 + r) * H + h) * DK + c;
                a = gate_logits ? gate_alpha(to_f32(static_cast<const Tin*>(alpha)[ia]))
                                : static_cast<const float*>(alpha)[ia];
            }
            if (a < 0.f) sg = -sg;
            L += log2f(fmaxf(fabsf(a), kFltMin));
            f.L[r * DK + c] = L;
            f.q[r * DK + c] *= sg;
            f.k[r * DK + c] *= sg;
        }
        f.sg[c] = sg;
        f.LC[c] = L;
    }
    __syncthreads();
    // A (strictly lower) and M (lower incl. diagonal)
    for (int e = tid; e < C * C; e += kThreads) {
        const int r = e / C, j = e % C;
        float a = 0.f, m = 0.f;
        if (j <= r) {
            for (int c = 0; c < DK; ++c) {
                const float kk = f.k[j * DK + c] * exp2f(f.L[r * DK + c] - f.L[j * DK + c]);
                a += f.k[r * DK + c] * kk;
                m += f.q[r * DK + c] * kk;
            }
            a = (j < r) ? a * f.b[r] : 0.f;
        }
        f.A[e] = a;
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
            acc += f.T[r * C + j] * f.b[j] * exp2f(f.L[j * DK + c]) * f.k[j * DK + c];
        f.W[e] = acc;
    }
    __syncthreads();
}

}  // namespace simt
}  // namespace ckda
