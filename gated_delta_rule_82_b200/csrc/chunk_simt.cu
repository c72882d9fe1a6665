// chunk_simt.cu -- chunked CKDA forward on CUDA cores, fp32 arithmetic (any supported size).
//
// Chunk algebra (derived from the transition of the "Complex KDA" paper summary, "Background":
// A_t = (I - beta_t k_t k_t^T) Diag(alpha_t)).  Inside a chunk of C tokens r = 0..C-1 with
// entering state S0, write gamma_r = prod_{tau<=r} alpha_tau (per channel).  Then
//     S_r = Diag(gamma_r) S0 + sum_{j<=r} Diag(gamma_r / gamma_j) k_j u_j^T
// where the pseudo-values u solve (I + A) U = diag(beta) (V - K_gamma S0) with
//     A_rj = beta_r k_r^T Diag(gamma_r/gamma_j) k_j  (j < r),   K_gamma,r = gamma_r * k_r.
// With T = (I + A)^-1 (unit lower triangular):  W = T diag(beta) K_gamma,  U~ = T diag(beta) V,
//     U   = U~ - W S0
//     O   = scale (Q_gamma S0 + M U),     M_rj = q_r^T Diag(gamma_r/gamma_j) k_j (j <= r)
//     S_C = Diag(gamma_C) S0 + K_end^T U, K_end,j = (gamma_C / gamma_j) * k_j.
//
// Signed gates: gamma is kept as a sign parity and a magnitude (the sign-magnitude split of
// Proposition 2 of the same page).  The parity sigma_r = prod sign(alpha_tau) is absorbed into
// q and k (q' = sigma q, k' = sigma k; the page's compiled-PyTorch variant), after which every
// ratio gamma_r/gamma_j becomes |gamma_r|/|gamma_j| = exp2(L_r - L_j) with L the running sum of
// log2 |alpha| from the chunk start.  Only non-positive exponents are ever evaluated (j <= r), so
// no 1/gamma is formed and nothing overflows; |alpha| is floored at FLT_MIN before the log (an
// exact zero gate leaves a factor below 1e-38).  The chunk-end state gets the parity back:
//     Diag(gamma_C) = Diag(sigma_C exp2(L_C)),   K_end,j = sigma_C exp2(L_C - L_j) k'_j.
//
// One CTA per (batch*head, dv slice): the slices of S are independent columns, so the chunk
// loop runs with no inter-CTA communication; the intra-chunk factors are recomputed per slice.
// This path favours plain, checkable loops over speed; the tensor-core path is the fast one.
#include "internal.cuh"

namespace ckda {

namespace {

constexpr int kSimtThreads = 256;

template <int DK, int DV, int C>
struct SimtShape {
    static constexpr int DVS = DV < 16 ? DV : 16;  // columns of S per CTA
    // shared memory layout (floats)
    static constexpr int off_q = 0;                 // q'      [C][DK]
    static constexpr int off_k = off_q + C * DK;    // k'      [C][DK]
    static constexpr int off_L = off_k + C * DK;    // L       [C][DK]
    static constexpr int off_W = off_L + C * DK;    // W       [C][DK]
    static constexpr int off_A = off_W + C * DK;    // A       [C][C]
    static constexpr int off_M = off_A + C * C;     // M       [C][C]
    static constexpr int off_T = off_M + C * C;     // T       [C][C]
    static constexpr int off_v = off_T + C * C;     // v       [C][DVS]
    static constexpr int off_Ut = off_v + C * DVS;  // U~      [C][DVS]
    static constexpr int off_U = off_Ut + C * DVS;  // U       [C][DVS]
    static constexpr int off_S = off_U + C * DVS;   // S slice [DK][DVS]
    static constexpr int off_b = off_S + DK * DVS;  // beta    [C]
    static constexpr int off_sg = off_b + C;        // sigma_C [DK]
    static constexpr int off_LC = off_sg + DK;      // L_C     [DK]
    static constexpr int total = off_LC + DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kSimtThreads)
chunk_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const void* __restrict__ alpha, const float* __restrict__ beta,
                  const float* __restrict__ h0, T* __restrict__ out, float* __restrict__ hT,
                  int T_len, const int* cu, int H, int G, int l2norm, RopeParams rp, float scale,
                  long long pos_offset, int gate_logits) {
    using Sh = SimtShape<DK, DV, C>;
    constexpr int DVS = Sh::DVS;
    extern __shared__ float smem[];
    float* sq = smem + Sh::off_q;
    float* sk = smem + Sh::off_k;
    float* sL = smem + Sh::off_L;
    float* sW = smem + Sh::off_W;
    float* sA = smem + Sh::off_A;
    float* sM = smem + Sh::off_M;
    float* sT = smem + Sh::off_T;
    float* sv = smem + Sh::off_v;
    float* sUt = smem + Sh::off_Ut;
    float* sU = smem + Sh::off_U;
    float* sS = smem + Sh::off_S;
    float* sb = smem + Sh::off_b;
    float* ssg = smem + Sh::off_sg;
    float* sLC = smem + Sh::off_LC;

    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    // the sequence's tokens on the token axis: batch row b, or packed sequence b (cu != nullptr:
    // tokens cu[b] .. cu[b + 1] - 1, rotary positions again from pos_offset)
    const size_t first = cu ? (size_t)cu[b] : (size_t)b * T_len;
    const int len = cu ? cu[b + 1] - cu[b] : T_len;
    const int n0 = blockIdx.y * DVS;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kSimtThreads / 32;

    // RoPE frequencies in shared memory (lanes index them per channel; a per-lane index
    // into the kernel-parameter array would serialise in the constant cache).  The barrier at the
    // top of the chunk loop publishes them.
    __shared__ unsigned long long sfreq[DK / 2];
    if (rp.enabled)
        for (int i = tid; i < DK / 2; i += kSimtThreads) sfreq[i] = rp.turns[i];

    // entering state slice
    for (int e = tid; e < DK * DVS; e += kSimtThreads) {
        int c = e / DVS, n = e % DVS;
        sS[e] = h0 ? h0[((size_t)bh * DK + c) * DV + n0 + n] : 0.f;
    }

    const int nchunks = (len + C - 1) / C;
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = ch * C;
        const int nvalid = min(C, len - t0);
        __syncthreads();
        // ---- load the chunk: q, k, v slice, beta (padding rows are identity steps) ----
        for (int e = tid; e < C * DK; e += kSimtThreads) {
            int r = e / DK, c = e % DK;
            float qv = 0.f, kv = 0.f;
            if (r < nvalid) {
                // value head h reads q/k head h / G (grouped value heads; G = 1 without grouping)
                size_t row = ((first + t0 + r) * H + h) / G;
                qv = to_f32(q[row * DK + c]);
                kv = to_f32(k[row * DK + c]);
            }
            sq[e] = qv;
            sk[e] = kv;
        }
        for (int e = tid; e < C * DVS; e += kSimtThreads) {
            int r = e / DVS, n = e % DVS;
            float vv = 0.f;
            if (r < nvalid) vv = to_f32(v[((first + t0 + r) * H + h) * DV + n0 + n]);
            sv[e] = vv;
        }
        for (int r = tid; r < C; r += kSimtThreads) {
            float bv = r < nvalid ? beta[(first + t0 + r) * H + h] : 0.f;
            if (r < nvalid && gate_logits) bv = gate_beta(bv);   // beta = 2 sigma(b)
            sb[r] = bv;
        }
        __syncthreads();

        // ---- prologue per row (one warp per row): rotation, then L2 norm ----
        for (int r = warp; r < nvalid; r += NW) {
            constexpr int PER = (DK + 31) / 32;
            float qr[PER], kr[PER];
            long long p = pos_offset + t0 + r;
#pragma unroll
            for (int m = 0; m < PER; ++m) {
                int c = lane + 32 * m;
                qr[m] = c < DK ? sq[r * DK + c] : 0.f;
                kr[m] = c < DK ? sk[r * DK + c] : 0.f;
                if (rp.enabled && c < rp.rot_dims) {   // the first rot_dims channels rotate
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
                    float qp = sq[r * DK + partner], kp = sk[r * DK + partner];
                    qr[m] = first ? qr[m] * cs - qp * sn : qr[m] * cs + qp * sn;
                    kr[m] = first ? kr[m] * cs - kp * sn : kr[m] * cs + kp * sn;
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
                int c = lane + 32 * m;
                if (c < DK) { sq[r * DK + c] = qr[m]; sk[r * DK + c] = kr[m]; }
            }
        }
        __syncthreads();

        // ---- gate prep: sign parity and log2-magnitude prefix per channel; absorb signs ----
        for (int c = tid; c < DK; c += kSimtThreads) {
            float L = 0.f, sg = 1.f;
            for (int r = 0; r < C; ++r) {
                float a = 1.f;
                if (r < nvalid) {
                    const size_t ia = ((first + t0 + r) * H + h) * DK + c;
                    // gate values (fp32), or logits in the activation type: alpha = 2 sigma(a) - 1
                    a = gate_logits ? gate_alpha(to_f32(static_cast<const T*>(alpha)[ia]))
                                    : static_cast<const float*>(alpha)[ia];
                }
                if (a < 0.f) sg = -sg;
                L += log2f(fmaxf(fabsf(a), 1.17549435e-38f));
                sL[r * DK + c] = L;
                sq[r * DK + c] *= sg;
                sk[r * DK + c] *= sg;
            }
            ssg[c] = sg;
            sLC[c] = L;
        }
        __syncthreads();

        // ---- A (strictly lower) and M (lower incl. diagonal) ----
        for (int e = tid; e < C * C; e += kSimtThreads) {
            int r = e / C, j = e % C;
            float a = 0.f, m = 0.f;
            if (j <= r) {
                for (int c = 0; c < DK; ++c) {
                    float ratio = exp2f(sL[r * DK + c] - sL[j * DK + c]);
                    float kk = sk[j * DK + c] * ratio;
                    a += sk[r * DK + c] * kk;
                    m += sq[r * DK + c] * kk;
                }
                a = (j < r) ? a * sb[r] : 0.f;
            }
            sA[e] = a;
            sM[e] = m;
        }
        __syncthreads();

        // ---- T = (I + A)^-1 by forward substitution, one column per thread ----
        for (int j = tid; j < C; j += kSimtThreads) {
            for (int r = 0; r < C; ++r) {
                float t;
                if (r < j) t = 0.f;
                else if (r == j) t = 1.f;
                else {
                    float acc = 0.f;
                    for (int m = j; m < r; ++m) acc += sA[r * C + m] * sT[m * C + j];
                    t = -acc;
                }
                sT[r * C + j] = t;
            }
        }
        __syncthreads();

        // ---- W = T diag(beta) K_gamma,  U~ = T diag(beta) V ----
        for (int e = tid; e < C * DK; e += kSimtThreads) {
            int r = e / DK, c = e % DK;
            float acc = 0.f;
            for (int j = 0; j <= r; ++j)
                acc += sT[r * C + j] * sb[j] * exp2f(sL[j * DK + c]) * sk[j * DK + c];
            sW[e] = acc;
        }
        for (int e = tid; e < C * DVS; e += kSimtThreads) {
            int r = e / DVS, n = e % DVS;
            float acc = 0.f;
            for (int j = 0; j <= r; ++j) acc += sT[r * C + j] * sb[j] * sv[j * DVS + n];
            sUt[e] = acc;
        }
        __syncthreads();

        // ---- U = U~ - W S0 ----
        for (int e = tid; e < C * DVS; e += kSimtThreads) {
            int r = e / DVS, n = e % DVS;
            float acc = sUt[e];
            for (int c = 0; c < DK; ++c) acc -= sW[r * DK + c] * sS[c * DVS + n];
            sU[e] = acc;
        }
        __syncthreads();

        // ---- O = scale (Q_gamma S0 + M U) ----
        for (int e = tid; e < C * DVS; e += kSimtThreads) {
            int r = e / DVS, n = e % DVS;
            if (r >= nvalid) continue;
            float acc = 0.f;
            for (int c = 0; c < DK; ++c) acc += exp2f(sL[r * DK + c]) * sq[r * DK + c] * sS[c * DVS + n];
            for (int j = 0; j <= r; ++j) acc += sM[r * C + j] * sU[j * DVS + n];
            out[((first + t0 + r) * H + h) * DV + n0 + n] = from_f32<T>(scale * acc);
        }
        __syncthreads();

        // ---- S <- Diag(gamma_C) S0 + K_end^T U ----
        for (int e = tid; e < DK * DVS; e += kSimtThreads) {
            int c = e / DVS, n = e % DVS;
            float LC = sLC[c];
            float acc = exp2f(LC) * sS[e];
            for (int r = 0; r < C; ++r) acc += exp2f(LC - sL[r * DK + c]) * sk[r * DK + c] * sU[r * DVS + n];
            sS[e] = ssg[c] * acc;
        }
    }
    __syncthreads();
    if (hT) {
        for (int e = tid; e < DK * DVS; e += kSimtThreads) {
            int c = e / DVS, n = e % DVS;
            hT[((size_t)bh * DK + c) * DV + n0 + n] = sS[e];
        }
    }
}

template <typename T, int DK, int DV, int C>
cudaError_t launch_simt_t(const void* q, const void* k, const void* v, const void* alpha,
                          const float* beta, const float* h0, void* out, float* hT, int B,
                          int T_len, const int* cu, int H, int G, int l2norm, const RopeParams& rp, float scale,
                          long long pos_offset, int gate_logits, cudaStream_t stream) {
    using Sh = SimtShape<DK, DV, C>;
    auto kern = chunk_simt_kernel<T, DK, DV, C>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Sh::bytes);
    if (e != cudaSuccess) return e;
    dim3 grid(B * H, DV / Sh::DVS);
    kern<<<grid, kSimtThreads, Sh::bytes, stream>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), alpha, beta,
        h0, static_cast<T*>(out), hT, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits);
    return cudaGetLastError();
}

template <typename T, int DK, int DV>
cudaError_t dispatch_chunk(int chunk, const void* q, const void* k, const void* v,
                           const void* alpha, const float* beta, const float* h0, void* out,
                           float* hT, int B, int T_len, const int* cu, int H, int G, int l2norm, const RopeParams& rp,
                           float scale, long long pos_offset, int gate_logits, cudaStream_t stream) {
    switch (chunk) {
        case 16: return launch_simt_t<T, DK, DV, 16>(q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
        case 32: return launch_simt_t<T, DK, DV, 32>(q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
        case 64: return launch_simt_t<T, DK, DV, 64>(q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename T, int DK>
cudaError_t dispatch_dv(int dv, int chunk, const void* q, const void* k, const void* v,
                        const void* alpha, const float* beta, const float* h0, void* out,
                        float* hT, int B, int T_len, const int* cu, int H, int G, int l2norm, const RopeParams& rp,
                        float scale, long long pos_offset, int gate_logits, cudaStream_t stream) {
    switch (dv) {
        case 16: return dispatch_chunk<T, DK, 16>(chunk, q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
        case 32: return dispatch_chunk<T, DK, 32>(chunk, q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
        case 64: return dispatch_chunk<T, DK, 64>(chunk, q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
        case 128: return dispatch_chunk<T, DK, 128>(chunk, q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t dispatch_dk(int dk, int dv, int chunk, const void* q, const void* k, const void* v,
                        const void* alpha, const float* beta, const float* h0, void* out,
                        float* hT, int B, int T_len, const int* cu, int H, int G, int l2norm, const RopeParams& rp,
                        float scale, long long pos_offset, int gate_logits, cudaStream_t stream) {
    switch (dk) {
        case 16: return dispatch_dv<T, 16>(dv, chunk, q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
        case 32: return dispatch_dv<T, 32>(dv, chunk, q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
        case 64: return dispatch_dv<T, 64>(dv, chunk, q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
        case 128: return dispatch_dv<T, 128>(dv, chunk, q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_chunk_simt(const void* q, const void* k, const void* v, const void* alpha,
                              const float* beta, const float* h0, void* out, float* hT, int B,
                              int T_len, int H, int G, int dk, int dv, int chunk, int l2norm,
                              const RopeParams& rp, float scale, long long pos_offset,
                              int gate_logits, ckda_dtype dtype, const PackedSeqs& pk,
                              cudaStream_t stream) {
    const int* cu = pk.cu;
    if (cu) B = pk.n;   // one CTA row per packed sequence
    if (dtype == CKDA_BF16)
        return dispatch_dk<__nv_bfloat16>(dk, dv, chunk, q, k, v, alpha, beta, h0, out, hT, B,
                                          T_len, cu, H, G, l2norm, rp, scale, pos_offset, gate_logits, stream);
    return dispatch_dk<float>(dk, dv, chunk, q, k, v, alpha, beta, h0, out, hT, B, T_len, cu, H, G,
                              l2norm, rp, scale, pos_offset, gate_logits, stream);
}

}  // namespace ckda
