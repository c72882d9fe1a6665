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
#include "simt_chunk.cuh"

namespace ckda {

namespace {

constexpr int kSimtThreads = simt::kThreads;

template <int DK, int DV, int C>
struct SimtShape {
    static constexpr int DVS = DV < 16 ? DV : 16;  // columns of S per CTA
    // shared memory layout (floats): the chunk factors, then the CTA's value columns
    static constexpr int off_v = simt::Factors<DK, C>::floats;   // v       [C][DVS]
    static constexpr int off_Ut = off_v + C * DVS;                // U~      [C][DVS]
    static constexpr int off_U = off_Ut + C * DVS;                // U       [C][DVS]
    static constexpr int off_S = off_U + C * DVS;                 // S slice [DK][DVS]
    static constexpr int total = off_S + DK * DVS;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// out and hT are nullable.
template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kSimtThreads)
chunk_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const void* __restrict__ alpha, const float* __restrict__ beta,
                  const float* __restrict__ h0, T* __restrict__ out, float* __restrict__ hT,
                  int T_len, const int* cu, int H, int G, int l2norm,
                  RopeParams rp, float scale, long long pos_offset, int gate_logits) {
    using Sh = SimtShape<DK, DV, C>;
    constexpr int DVS = Sh::DVS;
    extern __shared__ float smem[];
    simt::Factors<DK, C> f;
    f.bind(smem);
    constexpr int LD = simt::Factors<DK, C>::LD;
    float* sv = smem + Sh::off_v;
    float* sUt = smem + Sh::off_Ut;
    float* sU = smem + Sh::off_U;
    float* sS = smem + Sh::off_S;

    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    // the sequence's tokens on the token axis: batch row b, or packed sequence b (cu != nullptr:
    // tokens cu[b] .. cu[b + 1] - 1, rotary positions again from pos_offset)
    const size_t first = cu ? (size_t)cu[b] : (size_t)b * T_len;
    const int len = cu ? cu[b + 1] - cu[b] : T_len;
    const int n0 = blockIdx.y * DVS;
    const int tid = threadIdx.x;

    // RoPE frequencies in shared memory (lanes index them per channel; a per-lane index into the
    // kernel-parameter array would serialise in the constant cache).  The barriers inside the
    // chunk loop publish them.
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
        for (int e = tid; e < C * DVS; e += kSimtThreads) {
            int r = e / DVS, n = e % DVS;
            float vv = 0.f;
            if (r < nvalid) vv = to_f32(v[((first + t0 + r) * H + h) * DV + n0 + n]);
            sv[e] = vv;
        }
        // prologue, signs, log2 prefix, A, M, T, W (ends with a barrier)
        simt::chunk_factors<T, DK, C>(f, q, k, alpha, beta, first, t0, nvalid, H, h, G, l2norm, rp,
                                      sfreq, pos_offset + t0, gate_logits);

        // ---- U~ = T diag(beta) V ----
        for (int e = tid; e < C * DVS; e += kSimtThreads) {
            int r = e / DVS, n = e % DVS;
            float acc = 0.f;
            for (int j = 0; j <= r; ++j) acc += f.T[r * C + j] * f.b[j] * sv[j * DVS + n];
            sUt[e] = acc;
        }
        __syncthreads();

        // ---- U = U~ - W S0 ----
        for (int e = tid; e < C * DVS; e += kSimtThreads) {
            int r = e / DVS, n = e % DVS;
            float acc = sUt[e];
            for (int c = 0; c < DK; ++c) acc -= f.W[r * LD + c] * sS[c * DVS + n];
            sU[e] = acc;
        }
        __syncthreads();

        // ---- O = scale (Q_gamma S0 + M U) ----
        if (out) {
            for (int e = tid; e < C * DVS; e += kSimtThreads) {
                int r = e / DVS, n = e % DVS;
                if (r >= nvalid) continue;
                float acc = 0.f;
                for (int c = 0; c < DK; ++c) acc += exp2f(f.L[r * LD + c]) * f.q[r * LD + c] * sS[c * DVS + n];
                for (int j = 0; j <= r; ++j) acc += f.M[r * C + j] * sU[j * DVS + n];
                out[((first + t0 + r) * H + h) * DV + n0 + n] = from_f32<T>(scale * acc);
            }
            __syncthreads();
        }

        // ---- S <- Diag(gamma_C) S0 + K_end^T U ----
        for (int e = tid; e < DK * DVS; e += kSimtThreads) {
            int c = e / DVS, n = e % DVS;
            float LC = f.LC[c];
            float acc = exp2f(LC) * sS[e];
            for (int r = 0; r < C; ++r) acc += exp2f(LC - f.L[r * LD + c]) * f.k[r * LD + c] * sU[r * DVS + n];
            sS[e] = f.sg[c] * acc;
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
cudaError_t launch_simt_t(const SimtArgs& a, cudaStream_t stream) {
    using Sh = SimtShape<DK, DV, C>;
    auto kern = chunk_simt_kernel<T, DK, DV, C>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Sh::bytes);
    if (e != cudaSuccess) return e;
    dim3 grid(a.B * a.H, DV / Sh::DVS);
    kern<<<grid, kSimtThreads, Sh::bytes, stream>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
        a.alpha, a.beta, a.h0, static_cast<T*>(a.out), a.hT, a.T_len, a.cu, a.H, a.G,
        a.l2norm, a.rp, a.scale, a.pos_offset, a.gate_logits);
    return cudaGetLastError();
}

template <typename T, int DK, int DV>
cudaError_t dispatch_chunk(int chunk, const SimtArgs& a, cudaStream_t stream) {
    switch (chunk) {
        case 16: return launch_simt_t<T, DK, DV, 16>(a, stream);
        case 32: return launch_simt_t<T, DK, DV, 32>(a, stream);
        case 64: return launch_simt_t<T, DK, DV, 64>(a, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename T, int DK>
cudaError_t dispatch_dv(int dv, int chunk, const SimtArgs& a, cudaStream_t stream) {
    switch (dv) {
        case 16: return dispatch_chunk<T, DK, 16>(chunk, a, stream);
        case 32: return dispatch_chunk<T, DK, 32>(chunk, a, stream);
        case 64: return dispatch_chunk<T, DK, 64>(chunk, a, stream);
        case 128: return dispatch_chunk<T, DK, 128>(chunk, a, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t dispatch_dk(int dk, int dv, int chunk, const SimtArgs& a, cudaStream_t stream) {
    switch (dk) {
        case 16: return dispatch_dv<T, 16>(dv, chunk, a, stream);
        case 32: return dispatch_dv<T, 32>(dv, chunk, a, stream);
        case 64: return dispatch_dv<T, 64>(dv, chunk, a, stream);
        case 128: return dispatch_dv<T, 128>(dv, chunk, a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_chunk_simt(const SimtArgs& a, int dk, int dv, int chunk, ckda_dtype dtype,
                              cudaStream_t stream) {
    if (dtype == CKDA_BF16) return dispatch_dk<__nv_bfloat16>(dk, dv, chunk, a, stream);
    return dispatch_dk<float>(dk, dv, chunk, a, stream);
}

cudaError_t launch_chunk_simt(const void* q, const void* k, const void* v, const void* alpha,
                              const float* beta, const float* h0, void* out, float* hT, int B,
                              int T_len, int H, int G, int dk, int dv, int chunk, int l2norm,
                              const RopeParams& rp, float scale, long long pos_offset,
                              int gate_logits, ckda_dtype dtype, const PackedSeqs& pk,
                              cudaStream_t stream) {
    SimtArgs a{q, k, v, alpha, beta, h0, out, hT,
               pk.cu ? pk.n : B,   // one CTA row per packed sequence
               T_len, pk.cu, H, G, l2norm, rp, scale, pos_offset, gate_logits};
    return launch_chunk_simt(a, dk, dv, chunk, dtype, stream);
}

}  // namespace ckda
