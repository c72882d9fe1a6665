// chunk_bwd.cu -- gradients of the CKDA forward on CUDA cores (fp32): of L = <dout, out> +
// <dhT, hT> with respect to q, k, v, alpha, beta and h0.
//
// The backward runs the chunked form in reverse (derived from the transition of the "Complex
// KDA" paper summary, "Background"; the chunk factors are those of simt_chunk.cuh, with the gate
// signs absorbed into q' and k' and every gate ratio taken as R_rj = exp2(L_r - L_j) <= 1):
//   0. every chunk's factors are computed once, chunk-parallel, into a record in the workspace
//      (W, K_end, T, beta, gamma_C, Q', M and P = A before beta);
//   1. the forward replays the chunks from those records and keeps the state entering each one;
//   2. a chain over the chunks in reverse carries the gradient of the state:
//        dS_in = scale Q'^T dO + Diag(gamma_C) dS_out - W^T (K_end dS_out)
//      (Q' = Q_gamma - M W, K_end,j = sigma_C R_Cj k'_j), column slices of S independent;
//   3. every chunk then forms its input gradients from its record, its entering state, dS_out and
//      dO:
//        dQ' = scale dO S0^T,  dM = scale dO U^T - dQ' W^T,  dU = scale M^T dO + K_end dS_out,
//        dK_end = (U - W S0) dS_out^T,  dW = -(K_end dS_out) S0^T - M^T dQ',
//        dgamma_C = rowsum(dS_out . S0),  dT = dW (B K_gamma)^T + dU (B V)^T,
//        dA = strict_lower(-T^T dT T^T),  dV = B T^T dU,  dbeta from W, U and A,
//      then through the ratios to k', q' and the gate magnitudes.  The gate gradient needs no
//      division by alpha (exact zeros included):
//        dalpha_t = sign(alpha_t) [ g_{t-1} sum_{r>=t} dg_r R_rt + sum_{a>=t} R_at Z_at ],
//        Z_{a,t+1} = |alpha_t| Z_at + dR_at,  Z_a0 = 0,
//      where dg and dR are the gradients with respect to g_r = |gamma_r| and R_rj;
//   4. the prologue backward: the q/k gradients of a grouped head are summed over the value
//      heads it serves, then taken back through the L2 norm and the rotation (by -angle).
// The backward's chunk is 16 tokens (the gradients do not depend on it beyond rounding).
#include "simt_chunk.cuh"

namespace ckda {

namespace {

using simt::Factors;
using simt::kThreads;
constexpr int kBwdC = 16;

// ---- the record of a chunk's factors (fp32, rows DK floats apart) ----------------------------------
// [W | K_end | T | beta | gamma_C | Q' | M | P]: the replay reads the prefix up to Q', the chain up to
// M, the chunk gradients all of it.  Every offset is a multiple of 4 floats.
template <int DK, int C>
struct Rec {
    static constexpr int W = 0, KE = C * DK, T = 2 * C * DK, B = T + C * C, GC = B + C;
    static constexpr int QP = GC + DK, M = QP + C * DK, P = M + C * C, floats = P + C * C;
};

// 16-byte copies global -> shared on the load/store path, completed per thread by commit groups.
__device__ __forceinline__ void cp16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// the first `floats` floats of a chunk record into shared memory (one commit group)
__device__ __forceinline__ void load_record(float* dst, const float* src, int floats) {
    for (int i = threadIdx.x; i < floats / 4; i += kThreads) cp16(dst + 4 * i, src + 4 * i);
    cp_commit();
}

// ---- 0. every chunk's factors: one CTA per (b*h, chunk) -----------------------------------------
template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads)
bwd_factors_kernel(const T* __restrict__ q, const T* __restrict__ k, const void* __restrict__ alpha,
                   const float* __restrict__ beta, float* __restrict__ recs, int T_len, int H,
                   int G, int l2norm, RopeParams rp, long long pos_offset, int gate_logits) {
    using R = Rec<DK, C>;
    constexpr int LD = Factors<DK, C>::LD;
    extern __shared__ float smem[];
    Factors<DK, C> f;
    f.bind(smem);
    __shared__ unsigned long long sfreq[DK / 2];
    const int nchunks = (T_len + C - 1) / C;
    const int bh = blockIdx.x / nchunks, ch = blockIdx.x % nchunks;
    const int b = bh / H, h = bh % H;
    const int t0 = ch * C, nvalid = min(C, T_len - t0);
    const int tid = threadIdx.x;
    if (rp.enabled)
        for (int i = tid; i < DK / 2; i += kThreads) sfreq[i] = rp.turns[i];
    float* rec = recs + ((size_t)bh * nchunks + ch) * R::floats;
    simt::chunk_prep<T, DK, C>(f, q, k, alpha, beta, (size_t)b * T_len, t0, nvalid, H, h, G,
                               l2norm, rp, sfreq, pos_offset + t0, gate_logits);
    simt::chunk_products<DK, C>(f, rec + R::P);   // P = A before beta, straight to the record
    for (int e = tid; e < C * DK; e += kThreads) {
        const int r = e / DK, c = e % DK;
        float qp = exp2f(f.L[r * LD + c]) * f.q[r * LD + c];   // Q' = Q_gamma - M W
        for (int j = 0; j <= r; ++j) qp -= f.M[r * C + j] * f.W[j * LD + c];
        rec[R::W + e] = f.W[r * LD + c];
        rec[R::KE + e] = f.sg[c] * exp2f(f.LC[c] - f.L[r * LD + c]) * f.k[r * LD + c];
        rec[R::QP + e] = qp;
    }
    for (int e = tid; e < C * C; e += kThreads) {
        rec[R::T + e] = f.T[e];
        rec[R::M + e] = f.M[e];
    }
    for (int r = tid; r < C; r += kThreads) rec[R::B + r] = f.b[r];
    for (int c = tid; c < DK; c += kThreads) rec[R::GC + c] = f.sg[c] * exp2f(f.LC[c]);
}

// ---- 1. the forward replay: one CTA per (b*h, DVS columns of the state) ----------------------------
//   U~ = T B V,  U = U~ - W S,  S <- Diag(gamma_C) S + K_end^T U;  the state entering every chunk is
//   written to ws_S.  The next chunk's record is fetched while this one is used.
template <int DK, int DV, int C>
struct ReplayShape {
    static constexpr int DVS = DV < 16 ? DV : 16;
    static constexpr int REC = Rec<DK, C>::QP;               // the part of a record the replay reads
    static constexpr int off_v = 2 * REC;                    // two record stages, then V [C][DVS]
    static constexpr int off_ut = off_v + C * DVS;           // U~ [C][DVS]
    static constexpr int off_u = off_ut + C * DVS;           // U  [C][DVS]
    static constexpr int off_s = off_u + C * DVS;            // S  [DK][DVS]
    static constexpr int total = off_s + DK * DVS;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads)
bwd_replay_kernel(const T* __restrict__ v, const float* __restrict__ h0,
                  const float* __restrict__ recs, float* __restrict__ ws_S, int T_len, int H) {
    using R = Rec<DK, C>;
    using Sh = ReplayShape<DK, DV, C>;
    constexpr int DVS = Sh::DVS;
    extern __shared__ float smem[];
    float* sv = smem + Sh::off_v;
    float* sUt = smem + Sh::off_ut;
    float* sU = smem + Sh::off_u;
    float* sS = smem + Sh::off_s;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int n0 = blockIdx.y * DVS;
    const int tid = threadIdx.x;
    const int nchunks = (T_len + C - 1) / C;
    const float* rec0 = recs + (size_t)bh * nchunks * R::floats;
    for (int e = tid; e < DK * DVS; e += kThreads)
        sS[e] = h0 ? h0[((size_t)bh * DK + e / DVS) * DV + n0 + e % DVS] : 0.f;
    load_record(smem, rec0, Sh::REC);
    for (int ch = 0; ch < nchunks; ++ch) {
        const float* rf = smem + (ch & 1) * Sh::REC;
        if (ch + 1 < nchunks) {
            load_record(smem + ((ch + 1) & 1) * Sh::REC, rec0 + (size_t)(ch + 1) * R::floats, Sh::REC);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        const int t0 = ch * C, nvalid = min(C, T_len - t0);
        float* dst = ws_S + ((size_t)bh * nchunks + ch) * DK * DV + n0;
        for (int e = tid; e < DK * DVS; e += kThreads) dst[(e / DVS) * DV + e % DVS] = sS[e];
        for (int e = tid; e < C * DVS; e += kThreads) {
            const int r = e / DVS, n = e % DVS;
            sv[e] = r < nvalid ? to_f32(v[(((size_t)b * T_len + t0 + r) * H + h) * DV + n0 + n]) : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < C * DVS; e += kThreads) {
            const int r = e / DVS, n = e % DVS;
            float acc = 0.f;
            for (int j = 0; j <= r; ++j) acc += rf[R::T + r * C + j] * rf[R::B + j] * sv[j * DVS + n];
            sUt[e] = acc;
        }
        __syncthreads();
        for (int e = tid; e < C * DVS; e += kThreads) {
            const int r = e / DVS, n = e % DVS;
            float acc = sUt[e];
            for (int c = 0; c < DK; ++c) acc -= rf[R::W + r * DK + c] * sS[c * DVS + n];
            sU[e] = acc;
        }
        __syncthreads();
        for (int e = tid; e < DK * DVS; e += kThreads) {
            const int c = e / DVS, n = e % DVS;
            float acc = rf[R::GC + c] * sS[e];
            for (int r = 0; r < C; ++r) acc += rf[R::KE + r * DK + c] * sU[r * DVS + n];
            sS[e] = acc;
        }
        __syncthreads();   // this stage is refilled by the next iteration's prefetch
    }
}

// ---- 2. the state-gradient chain: one CTA per (b*h, DVS columns of the state) ----------------
template <int DK, int DV, int C>
struct ChainShape {
    static constexpr int DVS = DV < 16 ? DV : 16;
    static constexpr int REC = Rec<DK, C>::M;                 // the part of a record the chain reads
    static constexpr int off_do = 2 * REC;                    // two record stages, then dO [C][DVS]
    static constexpr int off_kd = off_do + C * DVS;           // K_end dS_out [C][DVS]
    static constexpr int off_ds = off_kd + C * DVS;           // dS_out [DK][DVS]
    static constexpr int total = off_ds + DK * DVS;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// ws_dS: [B*H][NT][DK][DV] fp32, the gradient with respect to each chunk's end state.
template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads)
bwd_chain_kernel(const T* __restrict__ dout, const float* __restrict__ dhT,
                 float* __restrict__ dh0, const float* __restrict__ recs, float* __restrict__ ws_dS,
                 int T_len, int H, float scale) {
    using R = Rec<DK, C>;
    using Sh = ChainShape<DK, DV, C>;
    constexpr int DVS = Sh::DVS;
    extern __shared__ float smem[];
    float* sdO = smem + Sh::off_do;
    float* sKd = smem + Sh::off_kd;
    float* sdS = smem + Sh::off_ds;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int n0 = blockIdx.y * DVS;
    const int tid = threadIdx.x;
    const int nchunks = (T_len + C - 1) / C;
    const float* rec0 = recs + (size_t)bh * nchunks * R::floats;
    for (int e = tid; e < DK * DVS; e += kThreads)
        sdS[e] = dhT ? dhT[((size_t)bh * DK + e / DVS) * DV + n0 + e % DVS] : 0.f;
    load_record(smem, rec0 + (size_t)(nchunks - 1) * R::floats, Sh::REC);
    for (int ch = nchunks - 1, it = 0; ch >= 0; --ch, ++it) {
        const float* rf = smem + (it & 1) * Sh::REC;
        if (ch > 0) {
            load_record(smem + ((it + 1) & 1) * Sh::REC, rec0 + (size_t)(ch - 1) * R::floats, Sh::REC);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        const int t0 = ch * C, nvalid = min(C, T_len - t0);
        float* dst = ws_dS + ((size_t)bh * nchunks + ch) * DK * DV + n0;
        for (int e = tid; e < DK * DVS; e += kThreads) dst[(e / DVS) * DV + e % DVS] = sdS[e];
        for (int e = tid; e < C * DVS; e += kThreads) {
            const int r = e / DVS, n = e % DVS;
            sdO[e] = r < nvalid ? to_f32(dout[(((size_t)b * T_len + t0 + r) * H + h) * DV + n0 + n]) : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < C * DVS; e += kThreads) {   // K_end dS_out
            const int j = e / DVS, n = e % DVS;
            float acc = 0.f;
            for (int c = 0; c < DK; ++c) acc += rf[R::KE + j * DK + c] * sdS[c * DVS + n];
            sKd[e] = acc;
        }
        __syncthreads();
        // dS_in = scale Q'^T dO + Diag(gamma_C) dS_out - W^T (K_end dS_out)
        for (int e = tid; e < DK * DVS; e += kThreads) {
            const int c = e / DVS, n = e % DVS;
            float acc = rf[R::GC + c] * sdS[e];
            for (int r = 0; r < C; ++r)
                acc += scale * rf[R::QP + r * DK + c] * sdO[r * DVS + n] - rf[R::W + r * DK + c] * sKd[r * DVS + n];
            sdS[e] = acc;   // each element is read only by its own thread above
        }
        __syncthreads();   // this stage is refilled by the next iteration's prefetch
    }
    if (dh0)
        for (int e = tid; e < DK * DVS; e += kThreads)
            dh0[((size_t)bh * DK + e / DVS) * DV + n0 + e % DVS] = sdS[e];
}

// ---- 3. the gradients of one chunk: one CTA per (b*h, chunk), all dv in tiles of DT ----------
template <int DK, int DV, int C>
struct GradShape {
    static constexpr int DT = DV < 32 ? DV : 32;
    static constexpr int TP = DT + 1;   // tile rows are TP floats apart (distinct banks down a column)
    static constexpr int CD = C * DK, CC = C * C, CT = C * TP;
    static constexpr int off_qp = Factors<DK, C>::floats;  // Q'     [C][DK]
    static constexpr int off_ke = off_qp + CD;             // K_end  [C][DK]
    static constexpr int off_dqp = off_ke + CD;            // dQ'    [C][DK]
    static constexpr int off_dke = off_dqp + CD;           // dK_end [C][DK]
    static constexpr int off_dw = off_dke + CD;            // dW, then dK_gamma [C][DK]
    static constexpr int off_sig = off_dw + CD;            // sigma  [C][DK]
    static constexpr int off_dgc = off_sig + CD;           // dgamma_C [DK]
    static constexpr int off_P = off_dgc + DK;             // P (A before beta) [C][C]
    static constexpr int off_dM = off_P + CC;              // dM [C][C]
    static constexpr int off_dT = off_dM + CC;             // dT, then E = B dA [C][C]
    static constexpr int off_Z = off_dT + CC;              // dT T^T [C][C]
    static constexpr int off_db = off_Z + CC;              // dbeta [C]
    static constexpr int off_s0 = off_db + C;              // S0 tile      [DK][TP]
    static constexpr int off_ds = off_s0 + DK * TP;        // dS_out tile  [DK][TP]
    static constexpr int off_do = off_ds + DK * TP;        // dO tile [C][TP]
    static constexpr int off_v = off_do + CT;              // V tile
    static constexpr int off_u = off_v + CT;               // U tile
    static constexpr int off_du = off_u + CT;              // dU tile
    static constexpr int off_ws = off_du + CT;             // W S0 tile
    static constexpr int off_kd = off_ws + CT;             // K_end dS_out tile
    static constexpr int total = off_kd + CT;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// recs: the chunk records; ws_S, ws_dS: [B*H][NT][DK][DV] fp32 (entering state, end-state
// gradient of each chunk); ws_dq, ws_dk: [B*T*H][DK] fp32 gradients of the prepared q^, k^ per
// value head.
template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads)
bwd_grad_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const void* __restrict__ alpha, const float* __restrict__ beta,
                const T* __restrict__ dout, const float* __restrict__ recs,
                const float* __restrict__ ws_S, const float* __restrict__ ws_dS,
                float* __restrict__ ws_dq,
                float* __restrict__ ws_dk, float* __restrict__ dv_out,
                float* __restrict__ dalpha, float* __restrict__ dbeta, int T_len, int H, int G,
                int l2norm, RopeParams rp, float scale, long long pos_offset, int gate_logits) {
    using Sh = GradShape<DK, DV, C>;
    constexpr int DT = Sh::DT;
    constexpr int TP = Sh::TP;   // padded row stride of the tiles
    constexpr int LD = Factors<DK, C>::LD;
    extern __shared__ float smem[];
    Factors<DK, C> f;
    f.bind(smem);
    float* sQp = smem + Sh::off_qp;
    float* sKe = smem + Sh::off_ke;
    float* sdQp = smem + Sh::off_dqp;
    float* sdKe = smem + Sh::off_dke;
    float* sdW = smem + Sh::off_dw;
    float* sSig = smem + Sh::off_sig;
    float* sdgC = smem + Sh::off_dgc;
    float* sP = smem + Sh::off_P;
    float* sdM = smem + Sh::off_dM;
    float* sdT = smem + Sh::off_dT;
    float* sZ = smem + Sh::off_Z;
    float* sdb = smem + Sh::off_db;
    float* tS0 = smem + Sh::off_s0;
    float* tdS = smem + Sh::off_ds;
    float* tdO = smem + Sh::off_do;
    float* tV = smem + Sh::off_v;
    float* tU = smem + Sh::off_u;
    float* tdU = smem + Sh::off_du;
    float* tWS = smem + Sh::off_ws;
    float* tKd = smem + Sh::off_kd;
    __shared__ unsigned long long sfreq[DK / 2];

    const int nchunks = (T_len + C - 1) / C;
    const int bh = blockIdx.x / nchunks, ch = blockIdx.x % nchunks;
    const int b = bh / H, h = bh % H;
    const int t0 = ch * C, nvalid = min(C, T_len - t0);
    const int tid = threadIdx.x;
    const size_t first = (size_t)b * T_len;
    if (rp.enabled)
        for (int i = tid; i < DK / 2; i += kThreads) sfreq[i] = rp.turns[i];
    // the record's T, M, P, Q' and K_end land while the chunk's rows are prepared; W goes to its
    // padded rows through registers
    {
        using R = Rec<DK, C>;
        const float* rec = recs + ((size_t)bh * nchunks + ch) * R::floats;
        for (int i = tid; i < C * C / 4; i += kThreads) {
            cp16(f.T + 4 * i, rec + R::T + 4 * i);
            cp16(f.M + 4 * i, rec + R::M + 4 * i);
            cp16(sP + 4 * i, rec + R::P + 4 * i);
        }
        for (int i = tid; i < C * DK / 4; i += kThreads) {
            cp16(sQp + 4 * i, rec + R::QP + 4 * i);
            cp16(sKe + 4 * i, rec + R::KE + 4 * i);
        }
        cp_commit();
        for (int e = tid; e < C * DK; e += kThreads) f.W[(e / DK) * LD + e % DK] = rec[R::W + e];
    }
    simt::chunk_prep<T, DK, C>(f, q, k, alpha, beta, first, t0, nvalid, H, h, G, l2norm, rp,
                               sfreq, pos_offset + t0, gate_logits);
    cp_wait<0>();
    auto gate = [&](int r, int c) {   // alpha of row r < nvalid, channel c
        const size_t ia = ((first + t0 + r) * H + h) * DK + c;
        return gate_logits ? gate_alpha(to_f32(static_cast<const T*>(alpha)[ia]))
                           : static_cast<const float*>(alpha)[ia];
    };
    // the running sign products; zero the accumulators
    for (int e = tid; e < C * DK; e += kThreads) {
        sdQp[e] = 0.f;
        sdKe[e] = 0.f;
        sdW[e] = 0.f;
    }
    for (int c = tid; c < DK; c += kThreads) {
        float s = 1.f;
        for (int r = 0; r < C; ++r) {
            if (r < nvalid && gate(r, c) < 0.f) s = -s;
            sSig[r * DK + c] = s;
        }
        sdgC[c] = 0.f;
    }
    for (int e = tid; e < C * C; e += kThreads) {
        sdM[e] = 0.f;
        sdT[e] = 0.f;
    }
    for (int r = tid; r < C; r += kThreads) sdb[r] = 0.f;
    __syncthreads();

    const float* S0 = ws_S + ((size_t)bh * nchunks + ch) * DK * DV;
    const float* dS = ws_dS + ((size_t)bh * nchunks + ch) * DK * DV;
    for (int n0 = 0; n0 < DV; n0 += DT) {
        // tiles of S0, dS_out, dO, V; U = T B V
        for (int e = tid; e < DK * DT; e += kThreads) {
            const int c = e / DT, n = e % DT;
            tS0[c * TP + n] = S0[(size_t)c * DV + n0 + n];
            tdS[c * TP + n] = dS[(size_t)c * DV + n0 + n];
        }
        for (int e = tid; e < C * DT; e += kThreads) {
            const int r = e / DT, n = e % DT;
            const size_t o = ((first + t0 + r) * H + h) * DV + n0 + n;
            tdO[r * TP + n] = r < nvalid ? to_f32(dout[o]) : 0.f;
            tV[r * TP + n] = r < nvalid ? to_f32(v[o]) : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < C * DT; e += kThreads) {
            const int j = e / DT, n = e % DT;
            float u = 0.f, ws = 0.f, kd = 0.f;
            for (int m = 0; m <= j; ++m) u += f.T[j * C + m] * f.b[m] * tV[m * TP + n];
            for (int c = 0; c < DK; ++c) {
                ws += f.W[j * LD + c] * tS0[c * TP + n];
                kd += sKe[j * DK + c] * tdS[c * TP + n];
            }
            tU[j * TP + n] = u;
            tWS[j * TP + n] = ws;
            tKd[j * TP + n] = kd;
        }
        __syncthreads();
        // dU = scale M^T dO + K_end dS_out
        for (int e = tid; e < C * DT; e += kThreads) {
            const int j = e / DT, n = e % DT;
            float acc = tKd[j * TP + n];
            for (int r = j; r < C; ++r) acc += scale * f.M[r * C + j] * tdO[r * TP + n];
            tdU[j * TP + n] = acc;
        }
        __syncthreads();
        // accumulate dQ', dK_end, dW over the tile's columns
        for (int e = tid; e < C * DK; e += kThreads) {
            const int r = e / DK, c = e % DK;
            float aq = 0.f, ak = 0.f, aw = 0.f;
            for (int n = 0; n < DT; ++n) {
                aq += tdO[r * TP + n] * tS0[c * TP + n];
                ak += (tU[r * TP + n] - tWS[r * TP + n]) * tdS[c * TP + n];
                aw += tKd[r * TP + n] * tS0[c * TP + n];
            }
            sdQp[e] += scale * aq;
            sdKe[e] += ak;
            sdW[e] -= aw;
        }
        for (int c = tid; c < DK; c += kThreads) {
            float acc = 0.f;
            for (int n = 0; n < DT; ++n) acc += tdS[c * TP + n] * tS0[c * TP + n];
            sdgC[c] += acc;
        }
        // dM += scale dO U^T;  dT += dU (B V)^T
        for (int e = tid; e < C * C; e += kThreads) {
            const int r = e / C, j = e % C;
            float am = 0.f, at = 0.f;
            for (int n = 0; n < DT; ++n) {
                am += tdO[r * TP + n] * tU[j * TP + n];
                at += tdU[r * TP + n] * tV[j * TP + n];
            }
            sdM[e] += scale * am;
            sdT[e] += f.b[j] * at;
        }
        // Y = T^T dU:  dv = B Y, dbeta += rowsum(Y . V)
        for (int j = tid / DT; j < C; j += kThreads / DT) {
            const int n = tid % DT;
            float y = 0.f;
            for (int r = j; r < C; ++r) y += f.T[r * C + j] * tdU[r * TP + n];
            if (j < nvalid) dv_out[((first + t0 + j) * H + h) * DV + n0 + n] = f.b[j] * y;
            float yv = y * tV[j * TP + n];
            for (int o = DT / 2; o > 0; o >>= 1) yv += __shfl_xor_sync(0xffffffffu, yv, o);
            if (n == 0) sdb[j] += yv;
        }
        __syncthreads();
    }

    // Q' = Q_gamma - M W:  dM -= dQ' W^T,  dW -= M^T dQ'
    for (int e = tid; e < C * C; e += kThreads) {
        const int r = e / C, j = e % C;
        float acc = 0.f;
        for (int c = 0; c < DK; ++c) acc += sdQp[r * DK + c] * f.W[j * LD + c];
        sdM[e] = j <= r ? sdM[e] - acc : 0.f;   // M is lower triangular (diagonal included)
    }
    for (int e = tid; e < C * DK; e += kThreads) {
        const int j = e / DK, c = e % DK;
        float acc = 0.f;
        for (int r = j; r < C; ++r) acc += f.M[r * C + j] * sdQp[r * DK + c];
        sdW[e] -= acc;
    }
    __syncthreads();
    // W = T B K_gamma:  dT += dW (B K_gamma)^T
    for (int e = tid; e < C * C; e += kThreads) {
        const int r = e / C, j = e % C;
        float acc = 0.f;
        for (int c = 0; c < DK; ++c) acc += sdW[r * DK + c] * exp2f(f.L[j * LD + c]) * f.k[j * LD + c];
        sdT[e] += f.b[j] * acc;
    }
    __syncthreads();
    // X = T^T dW (kept in dW's place; dK_gamma = B X);  Z = dT T^T
    for (int c = tid; c < DK; c += kThreads) {
        float x[C];
#pragma unroll
        for (int j = 0; j < C; ++j) {
            float acc = 0.f;
            for (int r = j; r < C; ++r) acc += f.T[r * C + j] * sdW[r * DK + c];
            x[j] = acc;
        }
#pragma unroll
        for (int j = 0; j < C; ++j) sdW[j * DK + c] = x[j];
    }
    for (int e = tid; e < C * C; e += kThreads) {
        const int r = e / C, j = e % C;
        float acc = 0.f;
        for (int m = 0; m < C; ++m) acc += sdT[r * C + m] * f.T[j * C + m];
        sZ[e] = acc;
    }
    __syncthreads();
    // dA = strict_lower(-T^T Z) (into dT's place);  dbeta += rowsum(X . K_gamma)
    for (int e = tid; e < C * C; e += kThreads) {
        const int r = e / C, j = e % C;
        float acc = 0.f;
        if (j < r)
            for (int m = 0; m < C; ++m) acc -= f.T[m * C + r] * sZ[m * C + j];
        sdT[e] = acc;
    }
    for (int j = tid >> 5; j < C; j += kThreads / 32) {   // one warp per row, lanes over channels
        float acc = 0.f;
        for (int c = tid & 31; c < DK; c += 32)
            acc += sdW[j * DK + c] * exp2f(f.L[j * LD + c]) * f.k[j * LD + c];
        acc = warp_sum(acc);
        if ((tid & 31) == 0) sdb[j] += acc;
    }
    __syncthreads();
    // A = B P:  dbeta += rowsum(dA . P);  E = B dA (in place)
    for (int r = tid; r < C; r += kThreads) {
        float acc = 0.f;
        for (int j = 0; j < r; ++j) acc += sdT[r * C + j] * sP[r * C + j];
        sdb[r] += acc;
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += kThreads) sdT[e] *= f.b[e / C];
    __syncthreads();
    const float* sE = sdT;

    // dq^, dk^ of every row (signs taken back out of q', k'):
    //   dk'_j = sum_{m<j} E_jm R_jm k'_m + sum_{r>j} E_rj R_rj k'_r + sum_{r>=j} dM_rj R_rj q'_r
    //           + dK_gamma,j g_j + dK_end,j sigma_C R_{C-1,j}
    //   dq'_j = sum_{m<=j} dM_jm R_jm k'_m + dQ_gamma,j g_j          (dQ_gamma = dQ')
    for (int e = tid; e < C * DK; e += kThreads) {
        const int j = e / DK, c = e % DK;
        if (j >= nvalid) continue;
        const float Lj = f.L[j * LD + c];
        float dk = 0.f, dq = 0.f;
        for (int m = 0; m < j; ++m) {
            const float R = exp2f(Lj - f.L[m * LD + c]);
            dk += sE[j * C + m] * R * f.k[m * LD + c];
            dq += sdM[j * C + m] * R * f.k[m * LD + c];
        }
        dq += sdM[j * C + j] * f.k[j * LD + c];
        for (int r = j; r < C; ++r) {
            const float R = exp2f(f.L[r * LD + c] - Lj);
            dk += (sE[r * C + j] * f.k[r * LD + c] + sdM[r * C + j] * f.q[r * LD + c]) * R;
        }
        const float g = exp2f(Lj);
        dk += f.b[j] * sdW[e] * g + sdKe[e] * f.sg[c] * exp2f(f.LC[c] - Lj);
        dq += sdQp[e] * g;
        const size_t o = ((first + t0 + j) * H + h) * DK + c;
        ws_dq[o] = sSig[e] * dq;
        ws_dk[o] = sSig[e] * dk;
    }
    // dalpha, one thread per channel c, in the order t = 0 .. C-1:
    //   dg_r = dK_gamma,r k'_r + dQ_gamma,r q'_r (+ dgamma_C sigma_C at the last row)
    //   dR_ab = E_ab k'_a k'_b + dM_ab q'_a k'_b (+ dK_end,b sigma_C k'_b at a = C-1), b <= a
    //   dalpha_t = sign(alpha_t) [g_{t-1} sum_{r>=t} dg_r R_rt + sum_{a>=t} R_at Z_at],
    //   Z_{a,t} = |alpha_{t-1}| Z_{a,t-1} + dR_{a,t-1},  Z_{a,0} = 0
    for (int c = tid; c < DK; c += kThreads) {
        const float sC = f.sg[c];
        float Z[C];
#pragma unroll
        for (int a = 0; a < C; ++a) Z[a] = 0.f;
        auto dR = [&](int a, int bb) {
            float x = (sE[a * C + bb] * f.k[a * LD + c] + sdM[a * C + bb] * f.q[a * LD + c]) * f.k[bb * LD + c];
            if (a == C - 1) x += sdKe[bb * DK + c] * sC * f.k[bb * LD + c];
            return x;
        };
        auto dg = [&](int r) {
            float x = f.b[r] * sdW[r * DK + c] * f.k[r * LD + c] + sdQp[r * DK + c] * f.q[r * LD + c];
            if (r == C - 1) x += sdgC[c] * sC;
            return x;
        };
#pragma unroll
        for (int t = 0; t < C; ++t) {
            if (t > 0) {
                const float am = exp2f(f.L[(t - 1) * LD + c] - (t > 1 ? f.L[(t - 2) * LD + c] : 0.f));
#pragma unroll
                for (int a = 0; a < C; ++a) Z[a] = a >= t - 1 ? am * Z[a] + dR(a, t - 1) : 0.f;
            }
            const float Lt = f.L[t * LD + c];
            const float gprev = t > 0 ? exp2f(f.L[(t - 1) * LD + c]) : 1.f;
            float s1 = 0.f, s2 = 0.f;
#pragma unroll
            for (int r = 0; r < C; ++r) {
                if (r < t) continue;
                const float R = exp2f(f.L[r * LD + c] - Lt);
                s1 += dg(r) * R;
                s2 += Z[r] * R;
            }
            if (t < nvalid) {
                const float a = gate(t, c);
                float d = (a < 0.f ? -1.f : 1.f) * (gprev * s1 + s2);
                if (gate_logits) d *= 0.5f * (1.f - a * a);   // alpha = 2 sigma(a) - 1
                dalpha[((first + t0 + t) * H + h) * DK + c] = d;
            }
        }
    }
    for (int r = tid; r < nvalid; r += kThreads) {
        const float bt = f.b[r];   // beta = 2 sigma(b): dbeta / db = beta (1 - beta / 2)
        dbeta[(first + t0 + r) * H + h] = gate_logits ? sdb[r] * bt * (1.f - 0.5f * bt) : sdb[r];
    }
}

// ---- 4. the prologue backward: one warp per (token, q/k head), q then k ------------------------
// dq^, dk^ of the G value heads that share a q/k head are summed; then through x^ = y s with
// y = R x and s = (|y|^2 + eps)^(-1/2):  dy = s dx^ - s^3 (y . dx^) y,  dx = R^T dy.
template <typename T, int DK>
__global__ void __launch_bounds__(kThreads)
bwd_prologue_kernel(const T* __restrict__ q, const T* __restrict__ k,
                    const float* __restrict__ ws_dq, const float* __restrict__ ws_dk,
                    float* __restrict__ dq, float* __restrict__ dk, int T_len, int Hk, int G,
                    long long rows, int l2norm, RopeParams rp, long long pos_offset) {
    constexpr int PER = (DK + 31) / 32;
    const int lane = threadIdx.x & 31;
    const long long wid = (long long)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    if (wid >= 2 * rows) return;
    const bool isk = wid >= rows;
    const long long row = isk ? wid - rows : wid;   // (b, t, hk)
    const int t = (int)((row / Hk) % T_len);
    const T* x = (isk ? k : q) + row * DK;
    const float* gsrc = isk ? ws_dk : ws_dq;
    float y[PER], g[PER];
#pragma unroll
    for (int m = 0; m < PER; ++m) {
        const int c = lane + 32 * m;
        y[m] = c < DK ? to_f32(x[c]) : 0.f;
        float acc = 0.f;
        if (c < DK)
            for (int j = 0; j < G; ++j) acc += gsrc[(row * G + j) * DK + c];
        g[m] = acc;
    }
    const long long p = pos_offset + t;
    // z <- R(sgn * angle) z over the first rot_dims channels; the pair partner of channel c is
    // read, by shuffle, from the lane and slot that hold it
    auto rotate = [&](float* z, float sgn) {
        float out[PER];
#pragma unroll
        for (int m = 0; m < PER; ++m) {
            const int c = lane + 32 * m;
            const bool rot = rp.enabled && c < rp.rot_dims;
            int i = 0, partner = c;
            bool lo = true;
            if (rot) {
                if (rp.convention == 0) {
                    const int half = rp.rot_dims / 2;
                    i = c % half; lo = c < half; partner = lo ? c + half : c - half;
                } else {
                    i = c / 2; lo = (c & 1) == 0; partner = c ^ 1;
                }
            }
            float zp = 0.f;
#pragma unroll
            for (int mm = 0; mm < PER; ++mm) {
                const float val = __shfl_sync(0xffffffffu, z[mm], partner & 31);
                if ((partner >> 5) == mm) zp = val;
            }
            out[m] = z[m];
            if (rot) {
                float sn, cs;
                rope_sincos(p, rp.turns[i], &sn, &cs);
                sn *= sgn;
                out[m] = lo ? z[m] * cs - zp * sn : z[m] * cs + zp * sn;
            }
        }
#pragma unroll
        for (int m = 0; m < PER; ++m) z[m] = out[m];
    };
    rotate(y, 1.f);
    if (l2norm) {
        float ss = 0.f, yg = 0.f;
#pragma unroll
        for (int m = 0; m < PER; ++m) { ss += y[m] * y[m]; yg += y[m] * g[m]; }
        ss = warp_sum(ss);
        yg = warp_sum(yg);
        const float s = rsqrtf(ss + kL2Eps);
#pragma unroll
        for (int m = 0; m < PER; ++m) g[m] = s * g[m] - s * s * s * yg * y[m];
    }
    rotate(g, -1.f);
#pragma unroll
    for (int m = 0; m < PER; ++m) {
        const int c = lane + 32 * m;
        if (c < DK) (isk ? dk : dq)[row * DK + c] = g[m];
    }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename T, int DK, int DV>
cudaError_t launch_bwd_t(const BwdArgs& a, const BwdLayout& w, cudaStream_t stream) {
    constexpr int C = kBwdC;
    const int BH = a.B * a.H;
    const int nt = (a.T_len + C - 1) / C;
    const T* q = static_cast<const T*>(a.q);
    const T* k = static_cast<const T*>(a.k);
    const T* v = static_cast<const T*>(a.v);
    const T* dout = static_cast<const T*>(a.dout);
    // 0. every chunk's factors
    auto factors = bwd_factors_kernel<T, DK, DV, C>;
    constexpr size_t fbytes = sizeof(float) * Factors<DK, C>::floats;
    cudaError_t e = set_smem(factors, fbytes);
    if (e != cudaSuccess) return e;
    factors<<<(unsigned)((size_t)BH * nt), kThreads, fbytes, stream>>>(
        q, k, a.alpha, a.beta, w.records, a.T_len, a.H, a.G, a.l2norm, a.rp, a.pos_offset,
        a.gate_logits);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 1. the forward replay, keeping every chunk's entering state
    using RS = ReplayShape<DK, DV, C>;
    auto replay = bwd_replay_kernel<T, DK, DV, C>;
    if ((e = set_smem(replay, RS::bytes)) != cudaSuccess) return e;
    replay<<<dim3(BH, DV / RS::DVS), kThreads, RS::bytes, stream>>>(v, a.h0, w.records, w.states,
                                                                   a.T_len, a.H);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 2. the state-gradient chain
    using CS = ChainShape<DK, DV, C>;
    auto chain = bwd_chain_kernel<T, DK, DV, C>;
    if ((e = set_smem(chain, CS::bytes)) != cudaSuccess) return e;
    chain<<<dim3(BH, DV / CS::DVS), kThreads, CS::bytes, stream>>>(
        dout, a.dhT, a.dh0, w.records, w.dstates, a.T_len, a.H, a.scale);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 3. every chunk's gradients
    using GS = GradShape<DK, DV, C>;
    auto grad = bwd_grad_kernel<T, DK, DV, C>;
    if ((e = set_smem(grad, GS::bytes)) != cudaSuccess) return e;
    grad<<<(unsigned)((size_t)BH * nt), kThreads, GS::bytes, stream>>>(
        q, k, v, a.alpha, a.beta, dout, w.records, w.states, w.dstates, w.dq, w.dk, a.dv,
        a.dalpha, a.dbeta, a.T_len, a.H, a.G, a.l2norm, a.rp, a.scale, a.pos_offset,
        a.gate_logits);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 4. the prologue backward (and the sum over grouped value heads)
    const long long rows = (long long)a.B * a.T_len * (a.H / a.G);
    const long long warps = 2 * rows;
    bwd_prologue_kernel<T, DK><<<(unsigned)((warps + kThreads / 32 - 1) / (kThreads / 32)),
                                 kThreads, 0, stream>>>(
        q, k, w.dq, w.dk, a.dq_out, a.dk_out, a.T_len, a.H / a.G, a.G, rows, a.l2norm, a.rp,
        a.pos_offset);
    return cudaGetLastError();
}

template <typename T, int DK>
cudaError_t bwd_dispatch_dv(int dv, const BwdArgs& a, const BwdLayout& w, cudaStream_t stream) {
    switch (dv) {
        case 16: return launch_bwd_t<T, DK, 16>(a, w, stream);
        case 32: return launch_bwd_t<T, DK, 32>(a, w, stream);
        case 64: return launch_bwd_t<T, DK, 64>(a, w, stream);
        case 128: return launch_bwd_t<T, DK, 128>(a, w, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t bwd_dispatch(int dk, int dv, const BwdArgs& a, const BwdLayout& w,
                         cudaStream_t stream) {
    switch (dk) {
        case 16: return bwd_dispatch_dv<T, 16>(dv, a, w, stream);
        case 32: return bwd_dispatch_dv<T, 32>(dv, a, w, stream);
        case 64: return bwd_dispatch_dv<T, 64>(dv, a, w, stream);
        case 128: return bwd_dispatch_dv<T, 128>(dv, a, w, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

// Workspace of the backward: the factor record of every chunk of 16 tokens
// ([B*H][ceil(T/16)][3*16*dk + 3*16*16 + 16 + dk] fp32), the entering state and the end-state
// gradient of every chunk ([B*H][ceil(T/16)][dk][dv] fp32 each), then the gradients of the
// prepared q^ and k^ per value head ([B*T*H][dk] fp32 each); every part 256-byte aligned.
BwdLayout bwd_layout(void* ws, int B, int T_len, int H, int dk, int dv) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    constexpr size_t C = kBwdC;
    const size_t nt = (size_t)(T_len + kBwdC - 1) / kBwdC;
    const size_t rec = up((size_t)B * H * nt * (3 * C * dk + 3 * C * C + C + dk) * sizeof(float));
    const size_t st = up((size_t)B * H * nt * dk * dv * sizeof(float));
    const size_t gr = up((size_t)B * T_len * H * dk * sizeof(float));
    BwdLayout w;
    uint8_t* p = static_cast<uint8_t*>(ws);
    w.records = reinterpret_cast<float*>(p);
    w.states = reinterpret_cast<float*>(p + rec);
    w.dstates = reinterpret_cast<float*>(p + rec + st);
    w.dq = reinterpret_cast<float*>(p + rec + 2 * st);
    w.dk = reinterpret_cast<float*>(p + rec + 2 * st + gr);
    w.bytes = rec + 2 * st + 2 * gr;
    return w;
}

cudaError_t launch_chunk_bwd(const BwdArgs& a, int dk, int dv, void* workspace,
                             cudaStream_t stream) {
    const BwdLayout w = bwd_layout(workspace, a.B, a.T_len, a.H, dk, dv);
    if (a.dtype == CKDA_BF16) return bwd_dispatch<__nv_bfloat16>(dk, dv, a, w, stream);
    return bwd_dispatch<float>(dk, dv, a, w, stream);
}

}  // namespace ckda
