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
// Two forms.  Given a workspace (ckda_fwd_simt_workspace_bytes), every chunk's factors are formed
// once, chunk-parallel, into a record (chunk_records.cuh; chunks of 16 tokens), and one CTA per
// (batch*head, 16 state columns) walks the chunks with the records:
//     U~ = T B V,  U = U~ - W S,  O = scale (Q' S + M U~),  S <- Diag(gamma_C) S + K_end^T U,
// (Q' = Q_gamma - M W), the products as warp-level tensor-core tiles with split tf32 operands
// (fp32-grade).  Without one (and for packed sequences), one CTA per (batch*head, dv slice) walks
// the chunks and recomputes the chunk factors in plain fp32 loops per slice.
#include "chunk_records.cuh"
#include "simt_records.h"

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

// ---- the forward pass over the chunk records: one CTA per (b*h, 16 state columns) ----------------
template <int DK, int DV, int C>
struct PassShape {
    static constexpr int DVS = DV < 16 ? DV : 16;
    static constexpr int NT = DVS / 8;                      // 8-column tiles
    static constexpr int SP = DVS + 8;                      // rows of V, U~, parts, S (fragment banks)
    static constexpr int KQ = (8 / NT) < (DK / 8) ? (8 / NT) : (DK / 8);   // parts of the DK sums
    static constexpr int KC = DK / KQ;
    static constexpr int REC = Stage<DK, C>::floats_fwd;
    static constexpr int off_v = 2 * REC;                   // two stages, then V [C][SP]
    static constexpr int off_ut = off_v + C * SP;           // U~ [C][SP]
    static constexpr int off_u = off_ut + C * SP;           // parts of U [KQ][C][SP]
    static constexpr int off_o = off_u + KQ * C * SP;       // parts of Q' S [KQ][C][SP]
    static constexpr int off_s = off_o + KQ * C * SP;       // S [DK][SP]
    static constexpr int total = off_s + DK * SP;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads)
simt_pass_kernel(const T* __restrict__ v, const float* __restrict__ h0,
                 const float* __restrict__ recs, T* __restrict__ out, float* __restrict__ hT,
                 int T_len, int H, float scale) {
    using R = Rec<DK, C>;
    using St = Stage<DK, C>;
    using Sh = PassShape<DK, DV, C>;
    constexpr int DVS = Sh::DVS, NT = Sh::NT, SP = Sh::SP, RP = St::RP, KQ = Sh::KQ, KC = Sh::KC;
    extern __shared__ float smem[];
    float* sv = smem + Sh::off_v;
    float* sUt = smem + Sh::off_ut;
    float* sU = smem + Sh::off_u;
    float* sO = smem + Sh::off_o;
    float* sS = smem + Sh::off_s;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int n0 = blockIdx.y * DVS;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nchunks = (T_len + C - 1) / C;
    const float* rec0 = recs + (size_t)bh * nchunks * R::floats;
    for (int e = tid; e < DK * DVS; e += kThreads)
        sS[(e / DVS) * SP + e % DVS] = h0 ? h0[((size_t)bh * DK + e / DVS) * DV + n0 + e % DVS] : 0.f;
    load_stage<DK, C>(smem, rec0, true, true);
    // this thread's elements of a chunk's V slice, read one chunk ahead into registers
    constexpr int NE = (C * DVS + kThreads - 1) / kThreads;
    float rv[NE];
    auto load_v = [&](int ch) {
        const int t0 = ch * C, nvalid = min(C, T_len - t0);
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = tid + i * kThreads, r = e / DVS, n = e % DVS;
            rv[i] = e < C * DVS && r < nvalid
                        ? to_f32(v[(((size_t)b * T_len + t0 + r) * H + h) * DV + n0 + n]) : 0.f;
        }
    };
    load_v(0);
    for (int ch = 0; ch < nchunks; ++ch) {
        const float* rf = smem + (ch & 1) * Sh::REC;
        const int t0 = ch * C, nvalid = min(C, T_len - t0);
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = tid + i * kThreads;
            if (e < C * DVS) sv[(e / DVS) * SP + e % DVS] = rv[i];
        }
        if (ch + 1 < nchunks) {
            load_v(ch + 1);
            load_stage<DK, C>(smem + ((ch + 1) & 1) * Sh::REC, rec0 + (size_t)(ch + 1) * R::floats,
                              true, true);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncthreads();
        if (warp < NT * KQ) {
            // part kq of U = U~ - W S and of Q' S (state rows kq KC ..), and U~ = T B V (kq = 0)
            const int nt = warp % NT, kq = warp / NT;
            float cu[4] = {0.f, 0.f, 0.f, 0.f}, co[4] = {0.f, 0.f, 0.f, 0.f};
            if (kq == 0) {
                mma3_tile<C>(cu, [&](int m, int k) { return rf[St::T + m * C + k] * rf[St::B + k]; },
                             [&](int k, int n) { return sv[k * SP + 8 * nt + n]; }, lane);
                st_frag(sUt, SP, 8 * nt, cu, 1.f, lane);
            }
            mma3_tile<KC>(cu, [&](int m, int k) { return -rf[St::W + m * RP + kq * KC + k]; },
                          [&](int k, int n) { return sS[(kq * KC + k) * SP + 8 * nt + n]; }, lane);
            mma3_tile<KC>(co, [&](int m, int k) { return rf[St::QP + m * RP + kq * KC + k]; },
                          [&](int k, int n) { return sS[(kq * KC + k) * SP + 8 * nt + n]; }, lane);
            st_frag(sU + kq * C * SP, SP, 8 * nt, cu, 1.f, lane);
            st_frag(sO + kq * C * SP, SP, 8 * nt, co, 1.f, lane);
        }
        __syncthreads();
        auto parts = [&](const float* p, int r, int n) {
            float x = 0.f;
#pragma unroll
            for (int kq = 0; kq < KQ; ++kq) x += p[kq * C * SP + r * SP + n];
            return x;
        };
        // S <- Diag(gamma_C) S + K_end^T U ((DK / 16) x NT tiles, in place), and the output
        // O = scale (Q' S + M U~) (NT more tiles)
        for (int id = warp; id < (DK / 16) * NT + NT; id += kThreads / 32) {
            if (id < (DK / 16) * NT) {
                const int r0 = 16 * (id / NT), nt = id % NT, c0 = 8 * nt + 2 * t;
                float c[4];
                c[0] = rf[St::GC + r0 + g] * sS[(r0 + g) * SP + c0];
                c[1] = rf[St::GC + r0 + g] * sS[(r0 + g) * SP + c0 + 1];
                c[2] = rf[St::GC + r0 + g + 8] * sS[(r0 + g + 8) * SP + c0];
                c[3] = rf[St::GC + r0 + g + 8] * sS[(r0 + g + 8) * SP + c0 + 1];
                mma3_tile<C>(c, [&](int m, int k) { return rf[St::KE + k * RP + r0 + m]; },
                             [&](int k, int n) { return parts(sU, k, 8 * nt + n); }, lane);
                st_frag(sS + r0 * SP, SP, 8 * nt, c, 1.f, lane);
            } else {
                const int nt = id - (DK / 16) * NT, c0 = 8 * nt + 2 * t;
                float c[4] = {0.f, 0.f, 0.f, 0.f};
                mma3_tile<C>(c, [&](int m, int k) { return rf[St::M + m * C + k]; },
                             [&](int k, int n) { return sUt[k * SP + 8 * nt + n]; }, lane);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = g + 8 * hf;
                    if (r < nvalid) {
                        T* dst = out + (((size_t)b * T_len + t0 + r) * H + h) * DV + n0 + c0;
                        dst[0] = from_f32<T>(scale * (c[2 * hf] + parts(sO, r, c0)));
                        dst[1] = from_f32<T>(scale * (c[2 * hf + 1] + parts(sO, r, c0 + 1)));
                    }
                }
            }
        }
        __syncthreads();   // this stage is refilled by the next iteration's prefetch
    }
    if (hT)
        for (int e = tid; e < DK * DVS; e += kThreads)
            hT[((size_t)bh * DK + e / DVS) * DV + n0 + e % DVS] = sS[(e / DVS) * SP + e % DVS];
}

constexpr int kRecC = 16;   // chunk of the record form

template <typename T, int DK, int DV>
cudaError_t launch_simt_rec_t(const SimtArgs& a, void* workspace, cudaStream_t stream) {
    constexpr int C = kRecC;
    const int BH = a.B * a.H;
    const int nt = (a.T_len + C - 1) / C;
    float* recs = static_cast<float*>(workspace);
    auto records = chunk_records_kernel<T, DK, DV, C>;
    constexpr size_t fbytes = sizeof(float) * Factors<DK, C>::floats;
    cudaError_t e = cudaFuncSetAttribute(records, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fbytes);
    if (e != cudaSuccess) return e;
    records<<<(unsigned)((size_t)BH * nt), kThreads, fbytes, stream>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), a.alpha, a.beta, recs, a.T_len, a.H,
        a.G, a.l2norm, a.rp, a.pos_offset, a.gate_logits);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    using PS = PassShape<DK, DV, C>;
    auto pass = simt_pass_kernel<T, DK, DV, C>;
    if ((e = cudaFuncSetAttribute(pass, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PS::bytes)) !=
        cudaSuccess)
        return e;
    pass<<<dim3(BH, DV / PS::DVS), kThreads, PS::bytes, stream>>>(
        static_cast<const T*>(a.v), a.h0, recs, static_cast<T*>(a.out), a.hT, a.T_len, a.H, a.scale);
    return cudaGetLastError();
}

template <typename T, int DK>
cudaError_t rec_dispatch_dv(int dv, const SimtArgs& a, void* ws, cudaStream_t stream) {
    switch (dv) {
        case 16: return launch_simt_rec_t<T, DK, 16>(a, ws, stream);
        case 32: return launch_simt_rec_t<T, DK, 32>(a, ws, stream);
        case 64: return launch_simt_rec_t<T, DK, 64>(a, ws, stream);
        case 128: return launch_simt_rec_t<T, DK, 128>(a, ws, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t rec_dispatch(int dk, int dv, const SimtArgs& a, void* ws, cudaStream_t stream) {
    switch (dk) {
        case 16: return rec_dispatch_dv<T, 16>(dv, a, ws, stream);
        case 32: return rec_dispatch_dv<T, 32>(dv, a, ws, stream);
        case 64: return rec_dispatch_dv<T, 64>(dv, a, ws, stream);
        case 128: return rec_dispatch_dv<T, 128>(dv, a, ws, stream);
    }
    return cudaErrorInvalidValue;
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

// Workspace of the record form: the factor record of every chunk of 16 tokens,
// [B*H][ceil(T/16)][3*16*dk + 3*16*16 + 16 + dk] fp32.
size_t simt_records_bytes(int B, int T_len, int H, int dk) {
    constexpr size_t C = kRecC;
    const size_t nt = (size_t)(T_len + kRecC - 1) / kRecC;
    return (size_t)B * H * nt * (3 * C * dk + 3 * C * C + C + dk) * sizeof(float);
}

cudaError_t launch_chunk_simt_records(const SimtArgs& a, int dk, int dv, ckda_dtype dtype,
                                      void* workspace, cudaStream_t stream) {
    if (dtype == CKDA_BF16) return rec_dispatch<__nv_bfloat16>(dk, dv, a, workspace, stream);
    return rec_dispatch<float>(dk, dv, a, workspace, stream);
}

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
