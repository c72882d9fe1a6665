// chunk_bwd.cu -- gradients of the CKDA forward in fp32-grade arithmetic: of L = <dout, out> +
// <dhT, hT> with respect to q, k, v, alpha, beta and h0.  fp32 on the CUDA cores, and the dense
// products (one chunk is 16 rows) as warp-level tensor-core tiles with split tf32 operands.
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
#include "chunk_records.cuh"

namespace ckda {

namespace {

constexpr int kBwdC = 16;

// ---- 1. the forward replay: one CTA per (b*h, DVS columns of the state) ----------------------------
//   U = T B V - W S,  S <- Diag(gamma_C) S + K_end^T U  (warp tiles; the state entering every chunk
//   is written to ws_S).  The next chunk's record and V slice are fetched while this one is used.
template <int DK, int DV, int C>
struct ReplayShape {
    static constexpr int DVS = DV < 16 ? DV : 16;
    static constexpr int NT = DVS / 8;                      // 8-column tiles
    static constexpr int SP = DVS + 8;                      // rows of V, U, S (fragment banks)
    // the W S product is split over KQ ranges of the state rows (one warp tile each), whose parts
    // are summed where U is read
    static constexpr int KQ = (8 / NT) < (DK / 8) ? (8 / NT) : (DK / 8);
    static constexpr int KC = DK / KQ;
    static constexpr int REC = Stage<DK, C>::floats_replay;
    static constexpr int off_v = 2 * REC;                   // two stages, then V [C][SP]
    static constexpr int off_u = off_v + C * SP;            // parts of U [KQ][C][SP]
    static constexpr int off_s = off_u + KQ * C * SP;       // S  [DK][SP]
    static constexpr int total = off_s + DK * SP;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads)
bwd_replay_kernel(const T* __restrict__ v, const float* __restrict__ h0,
                  const float* __restrict__ recs, float* __restrict__ ws_S, int T_len, int H) {
    using R = Rec<DK, C>;
    using St = Stage<DK, C>;
    using Sh = ReplayShape<DK, DV, C>;
    constexpr int DVS = Sh::DVS, NT = Sh::NT, SP = Sh::SP, RP = St::RP, KQ = Sh::KQ, KC = Sh::KC;
    extern __shared__ float smem[];
    float* sv = smem + Sh::off_v;
    float* sU = smem + Sh::off_u;
    float* sS = smem + Sh::off_s;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int n0 = blockIdx.y * DVS;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nchunks = (T_len + C - 1) / C;
    const float* rec0 = recs + (size_t)bh * nchunks * R::floats;
    for (int e = tid; e < DK * DVS; e += kThreads)
        sS[(e / DVS) * SP + e % DVS] = h0 ? h0[((size_t)bh * DK + e / DVS) * DV + n0 + e % DVS] : 0.f;
    load_stage<DK, C>(smem, rec0, false);
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
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = tid + i * kThreads;
            if (e < C * DVS) sv[(e / DVS) * SP + e % DVS] = rv[i];
        }
        if (ch + 1 < nchunks) {
            load_v(ch + 1);
            load_stage<DK, C>(smem + ((ch + 1) & 1) * Sh::REC, rec0 + (size_t)(ch + 1) * R::floats, false);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        float* dst = ws_S + ((size_t)bh * nchunks + ch) * DK * DV + n0;
        for (int e = tid; e < DK * DVS; e += kThreads) dst[(e / DVS) * DV + e % DVS] = sS[(e / DVS) * SP + e % DVS];
        __syncthreads();
        if (warp < NT * KQ) {   // part kq of U = T B V - W S, columns 8 nt ..
            const int nt = warp % NT, kq = warp / NT;
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            if (kq == 0)
                mma3_tile<C>(c, [&](int m, int k) { return rf[St::T + m * C + k] * rf[St::B + k]; },
                             [&](int k, int n) { return sv[k * SP + 8 * nt + n]; }, lane);
            mma3_tile<KC>(c, [&](int m, int k) { return -rf[St::W + m * RP + kq * KC + k]; },
                          [&](int k, int n) { return sS[(kq * KC + k) * SP + 8 * nt + n]; }, lane);
            st_frag(sU + kq * C * SP, SP, 8 * nt, c, 1.f, lane);
        }
        __syncthreads();
        // the parts of U summed once (in the order kq = 0 ..), in place in part 0
        for (int e = tid; e < C * DVS; e += kThreads) {
            const int o = (e / DVS) * SP + e % DVS;
            float x = sU[o];
#pragma unroll
            for (int kq = 1; kq < KQ; ++kq) x += sU[kq * C * SP + o];
            sU[o] = x;
        }
        __syncthreads();
        auto u_at = [&](int r, int n) { return sU[r * SP + n]; };
        // S <- Diag(gamma_C) S + K_end^T U: (DK / 16) x NT tiles, each read and written in place
        for (int id = warp; id < (DK / 16) * NT; id += kThreads / 32) {
            const int r0 = 16 * (id / NT), c0 = 8 * (id % NT) + 2 * t;
            float c[4];
            c[0] = rf[St::GC + r0 + g] * sS[(r0 + g) * SP + c0];
            c[1] = rf[St::GC + r0 + g] * sS[(r0 + g) * SP + c0 + 1];
            c[2] = rf[St::GC + r0 + g + 8] * sS[(r0 + g + 8) * SP + c0];
            c[3] = rf[St::GC + r0 + g + 8] * sS[(r0 + g + 8) * SP + c0 + 1];
            mma3_tile<C>(c, [&](int m, int k) { return rf[St::KE + k * RP + r0 + m]; },
                         [&](int k, int n) { return u_at(k, 8 * (id % NT) + n); }, lane);
            st_frag(sS + r0 * SP, SP, 8 * (id % NT), c, 1.f, lane);
        }
        __syncthreads();   // this stage is refilled by the next iteration's prefetch
    }
}

// ---- 2. the state-gradient chain: one CTA per (b*h, DVS columns of the state) ----------------
//   K_d = K_end dS_out,  dS_in = Diag(gamma_C) dS_out + scale Q'^T dO - W^T K_d  (warp tiles)
template <int DK, int DV, int C>
struct ChainShape {
    static constexpr int DVS = DV < 16 ? DV : 16;
    static constexpr int NT = DVS / 8;
    static constexpr int SP = DVS + 8;
    static constexpr int KQ = (8 / NT) < (DK / 8) ? (8 / NT) : (DK / 8);   // as in the replay
    static constexpr int KC = DK / KQ;
    static constexpr int REC = Stage<DK, C>::floats_chain;
    static constexpr int off_do = 2 * REC;                    // two stages, then dO [C][SP]
    static constexpr int off_kd = off_do + C * SP;            // parts of K_end dS_out [KQ][C][SP]
    static constexpr int off_ds = off_kd + KQ * C * SP;       // dS_out [DK][SP]
    static constexpr int total = off_ds + DK * SP;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// ws_dS: [B*H][NT][DK][DV] fp32, the gradient with respect to each chunk's end state.
template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads)
bwd_chain_kernel(const T* __restrict__ dout, const float* __restrict__ dhT,
                 float* __restrict__ dh0, const float* __restrict__ recs, float* __restrict__ ws_dS,
                 int T_len, int H, float scale) {
    using R = Rec<DK, C>;
    using St = Stage<DK, C>;
    using Sh = ChainShape<DK, DV, C>;
    constexpr int DVS = Sh::DVS, NT = Sh::NT, SP = Sh::SP, RP = St::RP, KQ = Sh::KQ, KC = Sh::KC;
    extern __shared__ float smem[];
    float* sdO = smem + Sh::off_do;
    float* sKd = smem + Sh::off_kd;
    float* sdS = smem + Sh::off_ds;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int n0 = blockIdx.y * DVS;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nchunks = (T_len + C - 1) / C;
    const float* rec0 = recs + (size_t)bh * nchunks * R::floats;
    for (int e = tid; e < DK * DVS; e += kThreads)
        sdS[(e / DVS) * SP + e % DVS] = dhT ? dhT[((size_t)bh * DK + e / DVS) * DV + n0 + e % DVS] : 0.f;
    load_stage<DK, C>(smem, rec0 + (size_t)(nchunks - 1) * R::floats, true);
    // this thread's elements of a chunk's dO slice, read one chunk ahead into registers
    constexpr int NE = (C * DVS + kThreads - 1) / kThreads;
    float rdo[NE];
    auto load_do = [&](int ch) {
        const int t0 = ch * C, nvalid = min(C, T_len - t0);
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = tid + i * kThreads, r = e / DVS, n = e % DVS;
            rdo[i] = e < C * DVS && r < nvalid
                         ? to_f32(dout[(((size_t)b * T_len + t0 + r) * H + h) * DV + n0 + n]) : 0.f;
        }
    };
    load_do(nchunks - 1);
    for (int ch = nchunks - 1, it = 0; ch >= 0; --ch, ++it) {
        const float* rf = smem + (it & 1) * Sh::REC;
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = tid + i * kThreads;
            if (e < C * DVS) sdO[(e / DVS) * SP + e % DVS] = rdo[i];
        }
        if (ch > 0) {
            load_do(ch - 1);
            load_stage<DK, C>(smem + ((it + 1) & 1) * Sh::REC, rec0 + (size_t)(ch - 1) * R::floats, true);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        float* dst = ws_dS + ((size_t)bh * nchunks + ch) * DK * DV + n0;
        for (int e = tid; e < DK * DVS; e += kThreads) dst[(e / DVS) * DV + e % DVS] = sdS[(e / DVS) * SP + e % DVS];
        __syncthreads();
        if (warp < NT * KQ) {   // part kq of K_end dS_out, columns 8 nt ..
            const int nt = warp % NT, kq = warp / NT;
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            mma3_tile<KC>(c, [&](int m, int k) { return rf[St::KE + m * RP + kq * KC + k]; },
                          [&](int k, int n) { return sdS[(kq * KC + k) * SP + 8 * nt + n]; }, lane);
            st_frag(sKd + kq * C * SP, SP, 8 * nt, c, 1.f, lane);
        }
        __syncthreads();
        // the parts of K_end dS_out summed once (in the order kq = 0 ..), in place in part 0
        for (int e = tid; e < C * DVS; e += kThreads) {
            const int o = (e / DVS) * SP + e % DVS;
            float x = sKd[o];
#pragma unroll
            for (int kq = 1; kq < KQ; ++kq) x += sKd[kq * C * SP + o];
            sKd[o] = x;
        }
        __syncthreads();
        auto kd_at = [&](int r, int n) { return sKd[r * SP + n]; };
        // dS_in = Diag(gamma_C) dS_out + scale Q'^T dO - W^T K_d, tiles read and written in place
        for (int id = warp; id < (DK / 16) * NT; id += kThreads / 32) {
            const int r0 = 16 * (id / NT), nt = id % NT, c0 = 8 * nt + 2 * t;
            float c[4];
            c[0] = rf[St::GC + r0 + g] * sdS[(r0 + g) * SP + c0];
            c[1] = rf[St::GC + r0 + g] * sdS[(r0 + g) * SP + c0 + 1];
            c[2] = rf[St::GC + r0 + g + 8] * sdS[(r0 + g + 8) * SP + c0];
            c[3] = rf[St::GC + r0 + g + 8] * sdS[(r0 + g + 8) * SP + c0 + 1];
            mma3_tile<C>(c, [&](int m, int k) { return scale * rf[St::QP + k * RP + r0 + m]; },
                         [&](int k, int n) { return sdO[k * SP + 8 * nt + n]; }, lane);
            mma3_tile<C>(c, [&](int m, int k) { return -rf[St::W + k * RP + r0 + m]; },
                         [&](int k, int n) { return kd_at(k, 8 * nt + n); }, lane);
            st_frag(sdS + r0 * SP, SP, 8 * nt, c, 1.f, lane);
        }
        __syncthreads();   // this stage is refilled by the next iteration's prefetch
    }
    if (dh0)
        for (int e = tid; e < DK * DVS; e += kThreads)
            dh0[((size_t)bh * DK + e / DVS) * DV + n0 + e % DVS] = sdS[(e / DVS) * SP + e % DVS];
}

// ---- 3. the gradients of one chunk: one CTA per (b*h, chunk), all dv in tiles of DT ----------
// The products over a dv tile are 16-row warp tiles (above): U, W S0, K_end dS_out, dU, and the
// accumulations dQ', dK_end, dW, dM, dT, whose fragments stay in registers across the dv tiles
// (tile q of the 3 DK/8 + 4 belongs to warp q % 8).
template <int DK, int DV, int C>
struct GradShape {
    static_assert(C == 16, "the warp tiles are 16 rows: one chunk");
    static constexpr int DT = 16;          // dv columns per tile
    static constexpr int NTT = DT / 8;     // 8-column tiles per dv tile
    static constexpr int TP = DT + 4;      // tile rows TP floats apart (fragment lanes on distinct banks)
    static constexpr int KP = DK + 4;      // rows of W, K_end and K_gamma (the same)
    static constexpr int NQ = 3 * (DK / 8) + 4;   // accumulated tiles: dQ', dK_end, dW, dM (2), dT (2)
    static constexpr int QI = (NQ + 7) / 8;       // of them per warp
    static constexpr int CD = C * DK, CC = C * C, CT = C * TP, CK = C * KP;
    static constexpr int off_w = Factors<DK, C>::floats_nw;  // W       [C][KP]
    static constexpr int off_ke = off_w + CK;              // K_end   [C][KP]
    static constexpr int off_kg = off_ke + CK;             // K_gamma [C][KP]
    static constexpr int off_al = off_kg + CK;             // alpha   [C][DK]
    static constexpr int off_sm = off_al + CD;             // running-sign bits per channel [DK]
    static constexpr int off_dgc = off_sm + DK;            // dgamma_C [DK]
    static constexpr int off_P = off_dgc + DK;             // P (A before beta) [C][C]
    static constexpr int off_dM = off_P + CC;              // dM [C][C]
    static constexpr int off_dT = off_dM + CC;             // dT, then E = B dA [C][C]
    static constexpr int off_Z = off_dT + CC;              // dT T^T [C][C]
    static constexpr int off_db = off_Z + CC;              // dbeta [C]
    static constexpr int off_yb = off_db + C;              // dbeta parts of the Y tiles [NTT][C]
    // the dv tiles; after the last one the same floats hold dQ', dK_end and dW (then X)
    static constexpr int off_tiles = off_yb + NTT * C;
    static constexpr int off_s0 = off_tiles;               // S0 tiles     [2][DK][TP]
    static constexpr int off_ds = off_s0 + 2 * DK * TP;    // dS_out tiles [2][DK][TP]
    static constexpr int off_do = off_ds + 2 * DK * TP;    // dO tile [C][TP]
    static constexpr int off_v = off_do + CT;              // V tile
    static constexpr int off_u = off_v + CT;               // U tile
    static constexpr int off_du = off_u + CT;              // dU tile
    static constexpr int off_ws = off_du + CT;             // W S0 tile
    static constexpr int off_kd = off_ws + CT;             // K_end dS_out tile
    static constexpr int off_dqp = off_tiles;              // dQ'    [C][DK]
    static constexpr int off_dke = off_dqp + CD;           // dK_end [C][DK]
    static constexpr int off_dw = off_dke + CD;            // dW, then X = T^T dW [C][DK]
    static constexpr int tiles_end = off_kd + CT, post_end = off_dw + CD;
    static constexpr int total = tiles_end > post_end ? tiles_end : post_end;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
    static_assert(off_tiles % 4 == 0 && off_w % 4 == 0 && (DK * TP) % 4 == 0,
                  "16-byte copies need 4-float offsets");
};

// recs: the chunk records; ws_S, ws_dS: [B*H][NT][DK][DV] fp32 (entering state, end-state
// gradient of each chunk); ws_dq, ws_dk: [B*T*H][DK] fp32 gradients of the prepared q^, k^ per
// value head.
template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads, 2)
bwd_grad_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const void* __restrict__ alpha, const float* __restrict__ beta,
                const T* __restrict__ dout, const float* __restrict__ recs,
                const float* __restrict__ ws_S, const float* __restrict__ ws_dS,
                float* __restrict__ ws_dq,
                float* __restrict__ ws_dk, float* __restrict__ dv_out,
                float* __restrict__ dalpha, float* __restrict__ dbeta, int T_len, int H, int G,
                int l2norm, RopeParams rp, float scale, long long pos_offset, int gate_logits) {
    using Sh = GradShape<DK, DV, C>;
    constexpr int DT = Sh::DT, NTT = Sh::NTT, NQ = Sh::NQ, QI = Sh::QI;
    constexpr int TP = Sh::TP, KP = Sh::KP;
    constexpr int LD = Factors<DK, C>::LD;
    constexpr int Q1 = DK / 8, Q2 = 2 * (DK / 8), Q3 = 3 * (DK / 8);   // tile-kind boundaries
    extern __shared__ float smem[];
    Factors<DK, C> f;
    f.bind_nw(smem);
    float* sW = smem + Sh::off_w;
    float* sKe = smem + Sh::off_ke;
    float* sKg = smem + Sh::off_kg;
    float* sdQp = smem + Sh::off_dqp;
    float* sdKe = smem + Sh::off_dke;
    float* sdW = smem + Sh::off_dw;
    uint32_t* sSgn = reinterpret_cast<uint32_t*>(smem + Sh::off_sm);
    float* sAl = smem + Sh::off_al;
    float* sdgC = smem + Sh::off_dgc;
    float* sP = smem + Sh::off_P;
    float* sdM = smem + Sh::off_dM;
    float* sdT = smem + Sh::off_dT;
    float* sZ = smem + Sh::off_Z;
    float* sdb = smem + Sh::off_db;
    float* sYb = smem + Sh::off_yb;
    float* tdO = smem + Sh::off_do;
    float* tV = smem + Sh::off_v;
    float* tU = smem + Sh::off_u;
    float* tdU = smem + Sh::off_du;
    float* tWS = smem + Sh::off_ws;
    float* tKd = smem + Sh::off_kd;
    // RoPE frequencies for the row preparation, in the second S0 tile buffer (first written by
    // the prefetch of the second dv tile, after the preparation); two CTAs of this kernel fit an
    // SM at dk = 128 only without a static array
    unsigned long long* sfreq = reinterpret_cast<unsigned long long*>(smem + Sh::off_s0 + DK * TP);

    const int nchunks = (T_len + C - 1) / C;
    const int bh = blockIdx.x / nchunks, ch = blockIdx.x % nchunks;
    const int b = bh / H, h = bh % H;
    const int t0 = ch * C, nvalid = min(C, T_len - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t first = (size_t)b * T_len;
    const float* S0 = ws_S + ((size_t)bh * nchunks + ch) * DK * DV;
    const float* dS = ws_dS + ((size_t)bh * nchunks + ch) * DK * DV;
    // the state tiles of dv columns n0 .. n0 + DT - 1 into buffer `buf` (one commit group)
    auto load_state_tiles = [&](int n0, int buf) {
        float* d0 = smem + Sh::off_s0 + buf * DK * TP;
        float* d1 = smem + Sh::off_ds + buf * DK * TP;
        for (int i = tid; i < DK * DT / 4; i += kThreads) {
            const int c = i / (DT / 4), n4 = 4 * (i % (DT / 4));
            cp16(d0 + c * TP + n4, S0 + (size_t)c * DV + n0 + n4);
            cp16(d1 + c * TP + n4, dS + (size_t)c * DV + n0 + n4);
        }
        cp_commit();
    };
    // this thread's elements of the dO and V tiles, read one tile ahead into registers
    constexpr int NE = (C * DT + kThreads - 1) / kThreads;
    float rdo[NE], rv[NE];
    auto load_act_tiles = [&](int n0) {
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = tid + i * kThreads, r = e / DT, n = e % DT;
            const size_t o = ((first + t0 + r) * H + h) * DV + n0 + n;
            const bool ok = e < C * DT && r < nvalid;
            rdo[i] = ok ? to_f32(dout[o]) : 0.f;
            rv[i] = ok ? to_f32(v[o]) : 0.f;
        }
    };
    if (rp.enabled)
        for (int i = tid; i < DK / 2; i += kThreads) sfreq[i] = rp.turns[i];
    // the record's W, K_end, T, M and P land while the chunk's rows are prepared again
    {
        using R = Rec<DK, C>;
        const float* rec = recs + ((size_t)bh * nchunks + ch) * R::floats;
        for (int i = tid; i < C * C / 4; i += kThreads) {
            cp16(f.T + 4 * i, rec + R::T + 4 * i);
            cp16(f.M + 4 * i, rec + R::M + 4 * i);
            cp16(sP + 4 * i, rec + R::P + 4 * i);
        }
        for (int i = tid; i < C * DK / 4; i += kThreads) {
            const int r = i / (DK / 4), c4 = 4 * (i % (DK / 4));
            cp16(sW + r * KP + c4, rec + R::W + r * DK + c4);
            cp16(sKe + r * KP + c4, rec + R::KE + r * DK + c4);
        }
        cp_commit();
    }
    load_state_tiles(0, 0);
    load_act_tiles(0);
    simt::chunk_prep<T, DK, C>(f, q, k, alpha, beta, first, t0, nvalid, H, h, G, l2norm, rp,
                               sfreq, pos_offset + t0, gate_logits, sAl);
    cp_wait<1>();   // the record (the first state tiles may still be in flight)
    // K_gamma = g k', the running sign products (bit r of a channel's word: negative through
    // row r); zero the dbeta parts
    for (int e = tid; e < C * DK; e += kThreads) {
        const int r = e / DK, c = e % DK;
        sKg[r * KP + c] = exp2f(f.L[r * LD + c]) * f.k[r * LD + c];
    }
    for (int c = tid; c < DK; c += kThreads) {
        uint32_t neg = 0, bits = 0;
        for (int r = 0; r < C; ++r) {
            if (sAl[r * DK + c] < 0.f) neg ^= 1u;
            bits |= neg << r;
        }
        sSgn[c] = bits;
    }
    for (int e = tid; e < NTT * C; e += kThreads) sYb[e] = 0.f;
    float dgc_acc = 0.f;   // dgamma_C of channel tid (tid < DK)
    float acc[QI][4];
#pragma unroll
    for (int i = 0; i < QI; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    __syncthreads();

    for (int n0 = 0, it = 0; n0 < DV; n0 += DT, ++it) {
        // this tile's dO and V from registers; the next tile's into registers and its state
        // tiles into the other buffer while this one is used
        const float* tS0 = smem + Sh::off_s0 + (it & 1) * DK * TP;
        const float* tdS = smem + Sh::off_ds + (it & 1) * DK * TP;
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = tid + i * kThreads, r = e / DT, n = e % DT;
            if (e < C * DT) {
                tdO[r * TP + n] = rdo[i];
                tV[r * TP + n] = rv[i];
            }
        }
        if (n0 + DT < DV) {
            load_act_tiles(n0 + DT);
            load_state_tiles(n0 + DT, (it + 1) & 1);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncthreads();
        // U = T B V (K = C), W S0 and K_end dS_out (K = DK): 3 NTT tiles
        for (int tt = warp; tt < 3 * NTT; tt += kThreads / 32) {
            const int kind = tt / NTT, nt = tt % NTT;
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            if (kind == 0) {
                mma3_tile<C>(c, [&](int m, int kk) { return f.T[m * C + kk] * f.b[kk]; },
                             [&](int kk, int n) { return tV[kk * TP + 8 * nt + n]; }, lane);
                st_frag(tU, TP, 8 * nt, c, 1.f, lane);
            } else if (kind == 1) {
                mma3_tile<DK>(c, [&](int m, int kk) { return sW[m * KP + kk]; },
                              [&](int kk, int n) { return tS0[kk * TP + 8 * nt + n]; }, lane);
                st_frag(tWS, TP, 8 * nt, c, 1.f, lane);
            } else {
                mma3_tile<DK>(c, [&](int m, int kk) { return sKe[m * KP + kk]; },
                              [&](int kk, int n) { return tdS[kk * TP + 8 * nt + n]; }, lane);
                st_frag(tKd, TP, 8 * nt, c, 1.f, lane);
            }
        }
        __syncthreads();
        // dU = K_end dS_out + scale M^T dO (NTT tiles); the accumulated tiles but dT; dgamma_C
        if (warp < NTT) {
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            mma3_tile<C>(c, [&](int m, int kk) { return f.M[kk * C + m]; },
                         [&](int kk, int n) { return tdO[kk * TP + 8 * warp + n]; }, lane);
            const int g = lane >> 2, t = lane & 3, col = 8 * warp + 2 * t;
            tdU[g * TP + col] = tKd[g * TP + col] + scale * c[0];
            tdU[g * TP + col + 1] = tKd[g * TP + col + 1] + scale * c[1];
            tdU[(g + 8) * TP + col] = tKd[(g + 8) * TP + col] + scale * c[2];
            tdU[(g + 8) * TP + col + 1] = tKd[(g + 8) * TP + col + 1] + scale * c[3];
        }
#pragma unroll
        for (int i = 0; i < QI; ++i) {
            const int qt = warp + 8 * i;
            if (qt < Q1) {                // dQ' += dO S0^T (scale at the end)
                mma3_tile<DT>(acc[i], [&](int m, int kk) { return tdO[m * TP + kk]; },
                              [&](int kk, int n) { return tS0[(8 * qt + n) * TP + kk]; }, lane);
            } else if (qt < Q2) {         // dK_end += (U - W S0) dS_out^T
                const int c0 = 8 * (qt - Q1);
                mma3_tile<DT>(acc[i], [&](int m, int kk) { return tU[m * TP + kk] - tWS[m * TP + kk]; },
                              [&](int kk, int n) { return tdS[(c0 + n) * TP + kk]; }, lane);
            } else if (qt < Q3) {         // -dW += (K_end dS_out) S0^T
                const int c0 = 8 * (qt - Q2);
                mma3_tile<DT>(acc[i], [&](int m, int kk) { return tKd[m * TP + kk]; },
                              [&](int kk, int n) { return tS0[(c0 + n) * TP + kk]; }, lane);
            } else if (qt < Q3 + 2) {     // dM += dO U^T (scale at the end)
                const int j0 = 8 * (qt - Q3);
                mma3_tile<DT>(acc[i], [&](int m, int kk) { return tdO[m * TP + kk]; },
                              [&](int kk, int n) { return tU[(j0 + n) * TP + kk]; }, lane);
            }
        }
        for (int c = tid; c < DK; c += kThreads) {
            float a = 0.f;
            for (int n = 0; n < DT; ++n) a += tdS[c * TP + n] * tS0[c * TP + n];
            dgc_acc += a;
        }
        __syncthreads();
        // dT += dU (B V)^T (its two tiles); Y = T^T dU (NTT tiles): dv = B Y, dbeta parts Y . V
#pragma unroll
        for (int i = 0; i < QI; ++i) {
            const int qt = warp + 8 * i;
            if (qt >= Q3 + 2 && qt < NQ) {
                const int j0 = 8 * (qt - Q3 - 2);
                mma3_tile<DT>(acc[i], [&](int m, int kk) { return tdU[m * TP + kk]; },
                              [&](int kk, int n) { return f.b[j0 + n] * tV[(j0 + n) * TP + kk]; },
                              lane);
            }
        }
        if (warp >= 8 - NTT) {
            const int nt = warp - (8 - NTT);
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            mma3_tile<C>(c, [&](int m, int kk) { return f.T[kk * C + m]; },
                         [&](int kk, int n) { return tdU[kk * TP + 8 * nt + n]; }, lane);
            const int g = lane >> 2, t = lane & 3, col = 8 * nt + 2 * t;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int j = g + 8 * hf;
                const float y0 = c[2 * hf], y1 = c[2 * hf + 1];
                if (j < nvalid)
                    *reinterpret_cast<float2*>(dv_out + ((first + t0 + j) * H + h) * DV + n0 + col) =
                        make_float2(f.b[j] * y0, f.b[j] * y1);
                float yv = y0 * tV[j * TP + col] + y1 * tV[j * TP + col + 1];
                yv += __shfl_xor_sync(0xffffffffu, yv, 1);
                yv += __shfl_xor_sync(0xffffffffu, yv, 2);
                if (t == 0) sYb[nt * C + j] += yv;
            }
        }
        __syncthreads();
    }
    // the accumulated tiles into shared memory: dQ' (scaled), dK_end, dW (negated), dM
    // (scaled), dT; dgamma_C; dbeta = the sum of the Y tiles' parts
#pragma unroll
    for (int i = 0; i < QI; ++i) {
        const int qt = warp + 8 * i;
        if (qt < Q1) st_frag(sdQp, DK, 8 * qt, acc[i], scale, lane);
        else if (qt < Q2) st_frag(sdKe, DK, 8 * (qt - Q1), acc[i], 1.f, lane);
        else if (qt < Q3) st_frag(sdW, DK, 8 * (qt - Q2), acc[i], -1.f, lane);
        else if (qt < Q3 + 2) st_frag(sdM, C, 8 * (qt - Q3), acc[i], scale, lane);
        else if (qt < NQ) st_frag(sdT, C, 8 * (qt - Q3 - 2), acc[i], 1.f, lane);
    }
    for (int c = tid; c < DK; c += kThreads) sdgC[c] = dgc_acc;
    for (int r = tid; r < C; r += kThreads) {
        float a = 0.f;
        for (int nt = 0; nt < NTT; ++nt) a += sYb[nt * C + r];
        sdb[r] = a;
    }
    __syncthreads();

    // Q' = Q_gamma - M W:  dM -= dQ' W^T,  dW -= M^T dQ'
    for (int e = tid; e < C * C; e += kThreads) {
        const int r = e / C, j = e % C;
        float acc = 0.f;
        for (int c = 0; c < DK; ++c) acc += sdQp[r * DK + c] * sW[j * KP + c];
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
        for (int c = 0; c < DK; ++c) acc += sdW[r * DK + c] * sKg[j * KP + c];
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
        for (int c = tid & 31; c < DK; c += 32) acc += sdW[j * DK + c] * sKg[j * KP + c];
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

    // The ratios R_rj = g_r / g_j of a chunk whose decay stays >= 2^-60 in every channel factor
    // into g_r and 1/g_j with room to spare in fp32 (products of a gradient and g stay normal), so
    // the sums over rows become warp-tile products and staircase sums; other chunks take the
    // ratios exactly, exp2(L_r - L_j) per channel.
    const bool factored = __syncthreads_and(tid >= DK || f.LC[tid] >= -60.f) != 0;
    if (factored) {
        static_assert(Sh::off_tiles + 3 * Sh::CD + 2 * Sh::CK <= Sh::total, "K/g, Q_gamma fit");
        // K / g and Q_gamma, rows KP apart, in the part of the tile region the loop left dead
        float* sKi = smem + Sh::off_tiles + 3 * Sh::CD;
        float* sQg = sKi + Sh::CK;
        for (int e = tid; e < C * DK; e += kThreads) {
            const int r = e / DK, c = e % DK;
            const float L = f.L[r * LD + c];
            sKi[r * KP + c] = f.k[r * LD + c] * exp2f(-L);
            sQg[r * KP + c] = f.q[r * LD + c] * exp2f(L);
        }
        __syncthreads();
        if (warp >= 4) {
            // dq^, dk^ on warp tiles of 8 channels (signs taken back out of q', k'):
            //   P1 = E (K/g),  P2 = E^T K_gamma + dM^T Q_gamma,  P3 = dM (K/g)
            //   dk'_j = g_j P1_j + P2_j / g_j + dK_gamma,j g_j + dK_end,j sigma_C g_C / g_j
            //   dq'_j = g_j (P3_j + dQ_gamma,j)
            const int g = lane >> 2, t = lane & 3;
            for (int id = warp - 4; id < DK / 8; id += kThreads / 32 - 4) {
                const int n0 = 8 * id;
                float p1[4] = {0.f, 0.f, 0.f, 0.f}, p2[4] = {0.f, 0.f, 0.f, 0.f};
                float p3[4] = {0.f, 0.f, 0.f, 0.f};
                mma3_tile<C>(p1, [&](int m, int kk) { return sE[m * C + kk]; },
                             [&](int kk, int n) { return sKi[kk * KP + n0 + n]; }, lane);
                mma3_tile<C>(p2, [&](int m, int kk) { return sE[kk * C + m]; },
                             [&](int kk, int n) { return sKg[kk * KP + n0 + n]; }, lane);
                mma3_tile<C>(p2, [&](int m, int kk) { return sdM[kk * C + m]; },
                             [&](int kk, int n) { return sQg[kk * KP + n0 + n]; }, lane);
                mma3_tile<C>(p3, [&](int m, int kk) { return sdM[m * C + kk]; },
                             [&](int kk, int n) { return sKi[kk * KP + n0 + n]; }, lane);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int j = g + 8 * hf, c = n0 + 2 * t;
                    if (j >= nvalid) continue;
                    float dq2[2], dk2[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int cc = c + u, i = 2 * hf + u;
                        const float L = f.L[j * LD + cc], gj = exp2f(L), hj = exp2f(-L);
                        const float sgn = (sSgn[cc] >> j) & 1u ? -1.f : 1.f;
                        dk2[u] = sgn * (gj * p1[i] + hj * p2[i] + f.b[j] * sdW[j * DK + cc] * gj +
                                        sdKe[j * DK + cc] * f.sg[cc] * exp2f(f.LC[cc] - L));
                        dq2[u] = sgn * gj * (p3[i] + sdQp[j * DK + cc]);
                    }
                    const size_t o = ((first + t0 + j) * H + h) * DK + c;
                    *reinterpret_cast<float2*>(ws_dq + o) = make_float2(dq2[0], dq2[1]);
                    *reinterpret_cast<float2*>(ws_dk + o) = make_float2(dk2[0], dk2[1]);
                }
            }
        } else if (tid < DK) {
            // dalpha of channel c = tid.  With D_ab = R_ab dR_ab = (K_gamma,a E_ab + Q_gamma,a dM_ab
            // (+ g_C sigma_C dK_end,b at a = C-1)) (K/g)_b and S_t = sum_{a>=t} sum_{b<t} D_ab
            // (the sum of R_at Z_at over a >= t, times g_t / g_{t-1}):
            //   dalpha_t = sign(alpha_t) (g_{t-1} / g_t) [sum_{r>=t} dg_r g_r + S_t]
            const int c = tid;
            float S[C];
#pragma unroll
            for (int b = 0; b < C; ++b) S[b] = 0.f;
            const float gC = exp2f(f.LC[c]) * f.sg[c];
#pragma unroll
            for (int a = 1; a < C; ++a) {
                const float ka = sKg[a * KP + c], qa = sQg[a * KP + c];
                float pr = 0.f;   // sum_{b < tt} D_ab
#pragma unroll
                for (int tt = 0; tt <= a; ++tt) {
                    S[tt] += pr;
                    if (tt < a) {
                        float d = ka * sE[a * C + tt] + qa * sdM[a * C + tt];
                        if (a == C - 1) d += gC * sdKe[tt * DK + c];
                        pr += d * sKi[tt * KP + c];
                    }
                }
            }
            float sfx = 0.f;   // sum_{r >= tt} dg_r g_r
#pragma unroll
            for (int tt = C - 1; tt >= 0; --tt) {
                const float L = f.L[tt * LD + c];
                float dg = f.b[tt] * sdW[tt * DK + c] * f.k[tt * LD + c] + sdQp[tt * DK + c] * f.q[tt * LD + c];
                if (tt == C - 1) dg += sdgC[c] * f.sg[c];
                sfx += dg * exp2f(L);
                if (tt < nvalid) {
                    const float Lp = tt > 0 ? f.L[(tt - 1) * LD + c] : 0.f;
                    const float a = sAl[tt * DK + c];
                    float d = (a < 0.f ? -1.f : 1.f) * exp2f(Lp - L) * (sfx + S[tt]);
                    if (gate_logits) d *= 0.5f * (1.f - a * a);   // alpha = 2 sigma(a) - 1
                    dalpha[((first + t0 + tt) * H + h) * DK + c] = d;
                }
            }
        }
    } else {

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
            const float sgn = (sSgn[c] >> j) & 1u ? -1.f : 1.f;
            ws_dq[o] = sgn * dq;
            ws_dk[o] = sgn * dk;
        }
        // dalpha in the order t = 0 .. C-1, two threads per channel c (lanes 2 c, 2 c + 1 of a warp),
        // thread half hh taking the rows a, r = hh mod 2 of the sums:
        //   dg_r = dK_gamma,r k'_r + dQ_gamma,r q'_r (+ dgamma_C sigma_C at the last row)
        //   dR_ab = E_ab k'_a k'_b + dM_ab q'_a k'_b (+ dK_end,b sigma_C k'_b at a = C-1), b <= a
        //   dalpha_t = sign(alpha_t) [g_{t-1} sum_{r>=t} dg_r R_rt + sum_{a>=t} R_at Z_at],
        //   Z_{a,t} = |alpha_{t-1}| Z_{a,t-1} + dR_{a,t-1},  Z_{a,0} = 0
        static_assert(2 * DK <= kThreads, "two threads per channel");
        if ((tid >> 1) < DK) {   // whole warps (DK is a multiple of 16)
            const int c = tid >> 1, hh = tid & 1;
            const float sC = f.sg[c];
            float Z[C / 2], dgv[C / 2];
    #pragma unroll
            for (int i = 0; i < C / 2; ++i) {
                const int r = 2 * i + hh;
                Z[i] = 0.f;
                dgv[i] = f.b[r] * sdW[r * DK + c] * f.k[r * LD + c] + sdQp[r * DK + c] * f.q[r * LD + c];
                if (r == C - 1) dgv[i] += sdgC[c] * sC;
            }
            auto dR = [&](int a, int bb) {
                float x = (sE[a * C + bb] * f.k[a * LD + c] + sdM[a * C + bb] * f.q[a * LD + c]) * f.k[bb * LD + c];
                if (a == C - 1) x += sdKe[bb * DK + c] * sC * f.k[bb * LD + c];
                return x;
            };
    #pragma unroll
            for (int t = 0; t < C; ++t) {
                if (t > 0) {
                    const float am = exp2f(f.L[(t - 1) * LD + c] - (t > 1 ? f.L[(t - 2) * LD + c] : 0.f));
    #pragma unroll
                    for (int i = 0; i < C / 2; ++i) {
                        const int a = 2 * i + hh;
                        Z[i] = a >= t - 1 ? am * Z[i] + dR(a, t - 1) : 0.f;
                    }
                }
                const float Lt = f.L[t * LD + c];
                float s1 = 0.f, s2 = 0.f;
    #pragma unroll
                for (int i = 0; i < C / 2; ++i) {
                    const int r = 2 * i + hh;
                    if (r < t) continue;
                    const float R = exp2f(f.L[r * LD + c] - Lt);
                    s1 += dgv[i] * R;
                    s2 += Z[i] * R;
                }
                s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
                s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
                if (hh == 0 && t < nvalid) {
                    const float gprev = t > 0 ? exp2f(f.L[(t - 1) * LD + c]) : 1.f;
                    const float a = sAl[t * DK + c];
                    float d = (a < 0.f ? -1.f : 1.f) * (gprev * s1 + s2);
                    if (gate_logits) d *= 0.5f * (1.f - a * a);   // alpha = 2 sigma(a) - 1
                    dalpha[((first + t0 + t) * H + h) * DK + c] = d;
                }
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
    auto factors = chunk_records_kernel<T, DK, DV, C>;
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
