// chunk_tc.cu -- chunked CKDA forward on the sm_100a tensor cores (bf16 q/k/v, dk = dv = 128,
// chunk C = 64), fp32 accumulation in Tensor Memory and an fp32 inter-chunk state.
//
// Chunk algebra (see chunk_simt.cu for the derivation from the transition of the "Complex KDA"
// paper summary, "Background").  For a chunk with entering state S0 and the per-channel gate
// products gamma_r = prod_{tau<=r} alpha_tau:
//     A_rj = beta_r k_r^T Diag(gamma_r/gamma_j) k_j (j < r),  M_rj = q_r^T Diag(gamma_r/gamma_j) k_j (j <= r)
//     T = (I + A)^-1,  W = T diag(beta) K_gamma,  U~ = T diag(beta) V
//     Q' = Q_gamma - M W,  O_loc = M U~                       (state-independent, chunk-parallel)
//     [O; U] = [scale (Q' S0 + O_loc); U~ - W S0],  S_C = Diag(gamma_C) S0 + K_end^T U   (serial)
//
// Gates.  The sign of gamma is a parity absorbed into q and k (q' = sigma q, k' = sigma k; the
// paper's compiled-PyTorch variant, sign-magnitude split of its Proposition 2), so that every
// ratio gamma_r/gamma_j (j <= r) becomes a product of |alpha| over (j, r].  Those products are
// formed block-locally on 16-row blocks, never by dividing chunk-long products:
//   fb_r  = prod |alpha| from the block start to r (inclusive)       <= 1
//   bb_j  = prod |alpha| over (j, block end]                          <= 1
//   P_I   = block total;  off-diagonal block (I > J):  ratio = fb_r * prod_{J<J'<I} P_J' * bb_j
// so both GEMM operands stay in [0, 1] and nothing overflows.  Inside a diagonal block the ratio
// is fb_r / fb_j, which is bounded by 2^60 when the block total is >= 2^-60 (always the case for
// gates with |alpha| >= 2^-3.75 on average); a block whose total is smaller (exact zeros, very
// strong decay) is recomputed exactly on CUDA cores with running products.
//
// Kernel 1 (ckda_tc_intra) -- one CTA per (chunk, batch*head), chunk-parallel:
//   q/k prologue (rotation by an angle recurrence, L2 norm from the unrotated row sums -- the
//   rotation preserves the norm), gate prep, operand tiles in swizzled shared memory, tcgen05
//   GEMMs for A and M (4 block-rows), T by blocked forward substitution in fp32, tcgen05 GEMMs for
//   [W | U~] = T' [K_gamma | V] and M [W | U~].  It writes, per chunk, UMMA-ready images of
//   [Q'; W] (128 x 128) and K_end^T (128 x 64), the dv tiles of U~ and O_loc, and gamma_C.
// Kernel 2 (ckda_tc_state) -- one CTA per (dv tile of 32 columns, batch*head), serial over chunks:
//   1-D bulk (TMA) copies of the chunk's images into a double-buffered stage, then
//   D1 = [Q'; W] S (tcgen05, M = 128, N = 32, K = 128), the epilogue turns D1 into O (written to
//   HBM) and U (written transposed to shared memory), D2 = K_end^T U (M = 128, N = 32, K = 64),
//   and the epilogue updates the fp32 master state held in registers, S = gamma_C * S + D2.
#include "internal.cuh"
#include "tc_sm100.cuh"

namespace ckda {

namespace {

constexpr int kC = 64, kDK = 128, kDV = 128, kDVT = 32, kNTile = kDV / kDVT;

// ---- workspace image of one chunk-head (bytes) ------------------------------------------------
constexpr uint32_t WS_QW = 0;         // [Q'; W] bf16, K-major swizzled, 128 rows x 128
constexpr uint32_t WS_KE = 32768;     // K_end^T bf16, K-major swizzled, 128 rows x 64
constexpr uint32_t WS_UO = 49152;     // per dv tile t: U~[64][32] bf16 then O_loc[64][32] bf16
constexpr uint32_t WS_G = 81920;      // gamma_C fp32 [128]
constexpr uint32_t WS_CHUNK = 82432;
constexpr uint32_t WS_UO_TILE = 8192;

// ---- kernel 1 shared memory (bytes from a 1024-aligned base) ---------------------------------
constexpr uint32_t P1_QF = 0;         // q' fp32 [64][128]; later Q_gamma
constexpr uint32_t P1_KF = 32768;     // k' fp32 [64][128]; later T fp32 [64][65], T' bf16, X
constexpr uint32_t P1_L = 65536;      // L tile bf16 K-major 128 x 128; later A fp32 [64][65], M bf16
constexpr uint32_t P1_B = 98304;      // B tiles (16+32+48+64 rows x 128); later [W|U~] MN-major
constexpr uint32_t P1_KV = 139264;    // [K_gamma | V] MN-major, 64 K-rows x 256
constexpr uint32_t P1_SM = 172032;    // small arrays
constexpr uint32_t P1_BYTES = P1_SM + 8192 + 1024;

constexpr uint32_t P1_T = P1_KF;              // fp32 [64][65]
constexpr uint32_t P1_TB = P1_KF + 17408;     // T' bf16 K-major 64 x 64 (8 KB)
constexpr uint32_t P1_X = P1_KF + 26624;      // fp32 [16][48]
constexpr uint32_t P1_A = P1_L;               // fp32 [64][65]
constexpr uint32_t P1_M = P1_L + 17408;       // M bf16 K-major 64 x 64 (8 KB)
constexpr uint32_t P1_WU = P1_B;              // [W | U~] MN-major 64 K-rows x 256 (32 KB)
__host__ __device__ constexpr uint32_t btile_off(int I) { return I == 0 ? 0u : I == 1 ? 4096u : I == 2 ? 12288u : 24576u; }
__host__ __device__ constexpr uint32_t amcol(int I) { return I == 0 ? 0u : I == 1 ? 16u : I == 2 ? 48u : 96u; }
constexpr int kStrideA = 65;

constexpr float kDiagSafe = 8.673617379884035e-19f;  // 2^-60

__device__ __forceinline__ void st_bf16(uint8_t* base, uint32_t off, float x) {
    *reinterpret_cast<__nv_bfloat16*>(base + off) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
// 8 floats -> one 16-byte chunk of bf16
__device__ __forceinline__ uint4 pack8(const float* x) {
    return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                      pack_bf16(x[6], x[7]));
}

__device__ int g_tc_error;  // nonzero after a bounded wait ran out (diagnostic)

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
}

__global__ void __launch_bounds__(256, 1)
ckda_tc_intra(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
              const __nv_bfloat16* __restrict__ v, const float* __restrict__ alpha,
              const float* __restrict__ beta, uint8_t* __restrict__ ws, int T_len, int H, int NT,
              int l2norm, RopeParams rp, long long pos_offset) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* QF = reinterpret_cast<float*>(sm + P1_QF);
    float* KF = reinterpret_cast<float*>(sm + P1_KF);
    float* gP = reinterpret_cast<float*>(sm + P1_SM);          // [4][128]
    float* gS = gP + 512;                                      // [4][128]
    float* red = gS + 512;                                     // [4][2][32]
    float* sb = red + 256;                                     // [64]
    int* unsafe = reinterpret_cast<int*>(sb + 64);             // [4]
    volatile int* abort_flag = unsafe + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(unsafe + 8);
    uint64_t* bar = reinterpret_cast<uint64_t*>(unsafe + 16);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ch = blockIdx.x % NT, bh = blockIdx.x / NT;
    const int b = bh / H, h = bh % H;
    const int t0 = ch * kC;
    const int nvalid = min(kC, T_len - t0);
    uint8_t* wsc = ws + ((size_t)bh * NT + ch) * WS_CHUNK;
    auto grow = [&](int r) -> size_t { return ((size_t)b * T_len + t0 + r) * H + h; };

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 256);
        tc::tmem_relinquish();
    }
    if (tid == 32) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    if (tid < 4) unsafe[tid] = 0;
    if (tid < 64) sb[tid] = tid < nvalid ? beta[grow(tid)] : 0.f;

    // ======== phase A: per-thread channel pair (ca, cb) x 16-row block I ========
    const int p = tid & 63, I = tid >> 6, r0 = 16 * I;
    const bool inter = rp.enabled && rp.convention == 1;
    const int ca = inter ? 2 * p : p, cb = inter ? 2 * p + 1 : p + 64;
    uint8_t* KV = sm + P1_KV;
    uint8_t* Lt = sm + P1_L;
    uint8_t* Bt = sm + P1_B;

    // V into the MN-major [K_gamma | V] tile (N offset 128)
#pragma unroll 4
    for (int rl = 0; rl < 16; ++rl) {
        int r = r0 + rl;
        float va = 0.f, vb = 0.f;
        if (r < nvalid) {
            va = bf16_at(v, grow(r) * kDV + ca);
            vb = bf16_at(v, grow(r) * kDV + cb);
        }
        st_bf16(KV, tc::sw128_mnmajor(r, 128 + ca, 64), va);
        st_bf16(KV, tc::sw128_mnmajor(r, 128 + cb, 64), vb);
    }

    float qa[16], qb[16], ka[16], kb[16];
#pragma unroll
    for (int rl = 0; rl < 16; ++rl) {
        int r = r0 + rl;
        if (r < nvalid) {
            size_t o = grow(r) * kDK;
            qa[rl] = bf16_at(q, o + ca); qb[rl] = bf16_at(q, o + cb);
            ka[rl] = bf16_at(k, o + ca); kb[rl] = bf16_at(k, o + cb);
        } else {
            qa[rl] = qb[rl] = ka[rl] = kb[rl] = 0.f;
        }
    }
    // row sums of squares (the rotation preserves them): transposed butterfly, lane l ends
    // with the warp total of value l (l < 16: q row l, else k row l - 16)
    {
        float x[32];
#pragma unroll
        for (int rl = 0; rl < 16; ++rl) {
            x[rl] = qa[rl] * qa[rl] + qb[rl] * qb[rl];
            x[16 + rl] = ka[rl] * ka[rl] + kb[rl] * kb[rl];
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < o; ++i) {
                float send = upper ? x[i] : x[i + o];
                float keep = upper ? x[i + o] : x[i];
                x[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        red[(I * 2 + (warp & 1)) * 32 + lane] = x[0];
    }
    if (rp.enabled) {
        const double om = rp.inv_freq[p];
        float sn, cs, s1, c1;
        rope_sincos(pos_offset + t0 + r0, om, &sn, &cs);
        rope_sincos(1, om, &s1, &c1);
#pragma unroll
        for (int rl = 0; rl < 16; ++rl) {
            float x0 = qa[rl], x1 = qb[rl];
            qa[rl] = x0 * cs - x1 * sn; qb[rl] = x1 * cs + x0 * sn;
            x0 = ka[rl]; x1 = kb[rl];
            ka[rl] = x0 * cs - x1 * sn; kb[rl] = x1 * cs + x0 * sn;
            float cn = cs * c1 - sn * s1;
            sn = sn * c1 + cs * s1;
            cs = cn;
        }
    }
    __syncthreads();
    if (l2norm) {
#pragma unroll
        for (int rl = 0; rl < 16; ++rl) {
            float sq = red[(I * 2) * 32 + rl] + red[(I * 2 + 1) * 32 + rl];
            float sk = red[(I * 2) * 32 + 16 + rl] + red[(I * 2 + 1) * 32 + 16 + rl];
            float fq = rsqrtf(sq + kL2Eps), fk = rsqrtf(sk + kL2Eps);
            qa[rl] *= fq; qb[rl] *= fq; ka[rl] *= fk; kb[rl] *= fk;
        }
    }

    // gates: block-prefix fb (inclusive), block-suffix bb (exclusive), block totals; the
    // block-local sign parity is absorbed into q and k at once
    float faa[16], fab[16], bba[16], bbb[16];
    {
        float aa[16], ab[16];
#pragma unroll
        for (int rl = 0; rl < 16; ++rl) {
            int r = r0 + rl;
            if (r < nvalid) {
                aa[rl] = alpha[grow(r) * kDK + ca];
                ab[rl] = alpha[grow(r) * kDK + cb];
            } else {
                aa[rl] = ab[rl] = 1.f;
            }
        }
        float pa = 1.f, pb = 1.f, sa = 1.f, sbb = 1.f;
#pragma unroll
        for (int rl = 0; rl < 16; ++rl) {
            pa *= fabsf(aa[rl]); pb *= fabsf(ab[rl]);
            sa = aa[rl] < 0.f ? -sa : sa;
            sbb = ab[rl] < 0.f ? -sbb : sbb;
            faa[rl] = pa; fab[rl] = pb;
            qa[rl] *= sa; ka[rl] *= sa; qb[rl] *= sbb; kb[rl] *= sbb;
        }
        float ba = 1.f, bbv = 1.f;
#pragma unroll
        for (int rl = 15; rl >= 0; --rl) {
            bba[rl] = ba; bbb[rl] = bbv;
            ba *= fabsf(aa[rl]); bbv *= fabsf(ab[rl]);
        }
        gP[I * 128 + ca] = pa; gP[I * 128 + cb] = pb;
        gS[I * 128 + ca] = sa; gS[I * 128 + cb] = sbb;
        if (!(pa >= kDiagSafe) || !(pb >= kDiagSafe)) unsafe[I] = 1;
    }
    __syncthreads();

    // cross-block prefixes: magnitude before / after this block, parity before it, totals
    float preA = 1.f, preB = 1.f, sufA = 1.f, sufB = 1.f, spA = 1.f, spB = 1.f;
    float allA = 1.f, allB = 1.f, salA = 1.f, salB = 1.f;
#pragma unroll
    for (int J = 0; J < 4; ++J) {
        float PA = gP[J * 128 + ca], PB = gP[J * 128 + cb];
        float SA = gS[J * 128 + ca], SB = gS[J * 128 + cb];
        allA *= PA; allB *= PB; salA *= SA; salB *= SB;
        if (J < I) { preA *= PA; preB *= PB; spA *= SA; spB *= SB; }
        if (J > I) { sufA *= PA; sufB *= PB; }
    }
    const bool diag_ok = !unsafe[I];
    float gA[16], gB[16];  // |gamma_r| for Q_gamma, kept until phase C
#pragma unroll
    for (int rl = 0; rl < 16; ++rl) {
        const int r = r0 + rl;
        const float qpa = spA * qa[rl], qpb = spB * qb[rl];
        const float kpa = spA * ka[rl], kpb = spB * kb[rl];
        QF[r * 128 + ca] = qpa; QF[r * 128 + cb] = qpb;
        KF[r * 128 + ca] = kpa; KF[r * 128 + cb] = kpb;
        // A/M left operands: rows 32I + rl (k) and 32I + 16 + rl (q)
        st_bf16(Lt, tc::sw128_kmajor(32 * I + rl, ca, 128), kpa * faa[rl]);
        st_bf16(Lt, tc::sw128_kmajor(32 * I + rl, cb, 128), kpb * fab[rl]);
        st_bf16(Lt, tc::sw128_kmajor(32 * I + 16 + rl, ca, 128), qpa * faa[rl]);
        st_bf16(Lt, tc::sw128_kmajor(32 * I + 16 + rl, cb, 128), qpb * fab[rl]);
        // right operand of the diagonal block I
        {
            const int n = 16 * (I + 1);
            float da = diag_ok ? kpa / faa[rl] : 0.f, db = diag_ok ? kpb / fab[rl] : 0.f;
            st_bf16(Bt + btile_off(I), tc::sw128_kmajor(r, ca, n), da);
            st_bf16(Bt + btile_off(I), tc::sw128_kmajor(r, cb, n), db);
        }
        // right operands of the off-diagonal blocks (I2 > I)
        float midA = 1.f, midB = 1.f;
#pragma unroll
        for (int I2 = 1; I2 < 4; ++I2) {
            if (I2 > I) {
                const int n = 16 * (I2 + 1);
                st_bf16(Bt + btile_off(I2), tc::sw128_kmajor(r, ca, n), kpa * bba[rl] * midA);
                st_bf16(Bt + btile_off(I2), tc::sw128_kmajor(r, cb, n), kpb * bbb[rl] * midB);
                midA *= gP[I2 * 128 + ca];
                midB *= gP[I2 * 128 + cb];
            }
        }
        gA[rl] = preA * faa[rl];
        gB[rl] = preB * fab[rl];
        st_bf16(KV, tc::sw128_mnmajor(r, ca, 64), gA[rl] * kpa);
        st_bf16(KV, tc::sw128_mnmajor(r, cb, 64), gB[rl] * kpb);
    }
    // K_end^T image: rows ca, cb; columns r0 .. r0 + 15 (two 16-byte chunks per row);
    // K_end,j = sigma_C (gamma_C / gamma_j) k'_j, from this thread's own k' values in KF
    {
        uint8_t* ke = wsc + WS_KE;
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
            float ea[8], eb[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int rl = 8 * hc + e;
                ea[e] = salA * sufA * bba[rl] * KF[(r0 + rl) * 128 + ca];
                eb[e] = salB * sufB * bbb[rl] * KF[(r0 + rl) * 128 + cb];
            }
            *reinterpret_cast<uint4*>(ke + tc::sw128_kmajor(ca, r0 + 8 * hc, 128)) = pack8(ea);
            *reinterpret_cast<uint4*>(ke + tc::sw128_kmajor(cb, r0 + 8 * hc, 128)) = pack8(eb);
        }
        if (I == 0) {
            float* G = reinterpret_cast<float*>(wsc + WS_G);
            G[ca] = salA * allA;
            G[cb] = salB * allB;
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ======== phase B: A and M block-rows on the tensor cores ========
    if (tid == 0) {
        const uint32_t l0 = tc::smem_u32(Lt), b0 = tc::smem_u32(Bt);
#pragma unroll
        for (int J = 0; J < 4; ++J) {
            const int n = 16 * (J + 1);
            const uint32_t idesc = tc::idesc_bf16_f32(64, n, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint64_t ad = tc::smem_desc_sw128(l0 + 4096 * J + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                uint64_t bd = tc::smem_desc_sw128(b0 + btile_off(J) + (ks >> 2) * n * 128 + (ks & 3) * 32, 16, 1024);
                tc::mma_bf16(tmem + amcol(J), ad, bd, idesc, ks > 0 ? 1u : 0u);
            }
        }
        tc::mma_commit(bar);
    }
    tc::mbar_wait(bar, 0, abort_flag);
    tc::tc_fence_after();
    float* sA = reinterpret_cast<float*>(sm + P1_A);
    uint8_t* sM = sm + P1_M;
    if (warp < 2) {
        // warp 0: lanes 0..15 hold the k rows (A); warp 1: lanes 32..47 hold the q rows (M)
        const int l = lane;
#pragma unroll
        for (int J = 0; J < 4; ++J) {
            const int r = 16 * J + (l & 15);
            const int n = 16 * (J + 1);
            for (int c0 = 0; c0 < n; c0 += 16) {
                float x[16];
                tc::tmem_ld16(tc::tmem_addr(tmem, 32 * warp, amcol(J) + c0), x);
                tc::tmem_ld_wait();
                if (l < 16) {
                    if (warp == 0) {
                        const float br = sb[r];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int j = c0 + i;
                            sA[r * kStrideA + j] = j < r ? br * x[i] : 0.f;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; i += 8) {
                            float y[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) y[e] = (c0 + i + e) <= r ? x[i + e] : 0.f;
                            *reinterpret_cast<uint4*>(sM + tc::sw128_kmajor(r, c0 + i, 64)) = pack8(y);
                        }
                    }
                }
            }
            if (l < 16) {
                for (int j = n; j < 64; j += 8) {
                    if (warp == 0) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) sA[r * kStrideA + j + e] = 0.f;
                    } else {
                        *reinterpret_cast<uint4*>(sM + tc::sw128_kmajor(r, j, 64)) = make_uint4(0, 0, 0, 0);
                    }
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();

    // exact recomputation of diagonal blocks whose gate total fell below 2^-60
    for (int J = 0; J < 4; ++J) {
        if (!unsafe[J]) continue;
        for (int pr = tid; pr < 136; pr += 256) {
            int rl = 0;
            while ((rl + 1) * (rl + 2) / 2 <= pr) ++rl;
            const int jl = pr - rl * (rl + 1) / 2;
            const int r = 16 * J + rl, j = 16 * J + jl;
            float accA = 0.f, accM = 0.f;
            for (int c = 0; c < kDK; ++c) {
                float f = 1.f;
                for (int tau = j + 1; tau <= r; ++tau)
                    f *= tau < nvalid ? fabsf(alpha[grow(tau) * kDK + c]) : 1.f;
                const float kj = KF[j * 128 + c] * f;
                accA += KF[r * 128 + c] * kj;
                accM += QF[r * 128 + c] * kj;
            }
            sA[r * kStrideA + j] = j < r ? sb[r] * accA : 0.f;
            st_bf16(sM, tc::sw128_kmajor(r, j, 64), accM);
        }
    }
    __syncthreads();

    // ======== phase C: T = (I + A)^-1 (fp32), T' = T diag(beta); Q_gamma in place of q' ========
    float* sT = reinterpret_cast<float*>(sm + P1_T);
    float* sX = reinterpret_cast<float*>(sm + P1_X);
#pragma unroll
    for (int rl = 0; rl < 16; ++rl) {
        QF[(r0 + rl) * 128 + ca] *= gA[rl];
        QF[(r0 + rl) * 128 + cb] *= gB[rl];
    }
    for (int e = tid; e < 64 * 64; e += 256) {
        const int r = e >> 6, j = e & 63;
        if ((j >> 4) > (r >> 4)) sT[r * kStrideA + j] = 0.f;
    }
    if (warp < 4 && lane < 16) {
        const int J = warp, l = lane, base = 16 * J;
        float tcol[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m)
                if (m < rr) acc += sA[(base + rr) * kStrideA + base + m] * tcol[m];
            tcol[rr] = rr < l ? 0.f : (rr == l ? 1.f : -acc);
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) sT[(base + rr) * kStrideA + base + l] = tcol[rr];
    }
    __syncthreads();
    for (int Ib = 1; Ib < 4; ++Ib) {
        const int ncol = 16 * Ib;
        for (int e = tid; e < 16 * ncol; e += 256) {
            const int rl = e / ncol, jj = e % ncol;
            const int Jb = jj >> 4;
            float x = 0.f;
            for (int m = 16 * Jb; m < 16 * Ib; ++m) x += sA[(16 * Ib + rl) * kStrideA + m] * sT[m * kStrideA + jj];
            sX[rl * 48 + jj] = x;
        }
        __syncthreads();
        for (int e = tid; e < 16 * ncol; e += 256) {
            const int rl = e / ncol, jj = e % ncol;
            float y = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) y += sT[(16 * Ib + rl) * kStrideA + 16 * Ib + m] * sX[m * 48 + jj];
            sT[(16 * Ib + rl) * kStrideA + jj] = -y;
        }
        __syncthreads();
    }
    uint8_t* sTb = sm + P1_TB;
    for (int e = tid; e < 64 * 8; e += 256) {
        const int r = e >> 3, j0 = (e & 7) * 8;
        float y[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = sT[r * kStrideA + j0 + i] * sb[j0 + i];
        *reinterpret_cast<uint4*>(sTb + tc::sw128_kmajor(r, j0, 64)) = pack8(y);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    // ======== phase D: [W | U~] = T' [K_gamma | V]  (M = 64, N = 256, K = 64) ========
    if (tid == 0) {
        const uint32_t a0 = tc::smem_u32(sTb), b0 = tc::smem_u32(KV);
        const uint32_t idesc = tc::idesc_bf16_f32(64, 256, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint64_t ad = tc::smem_desc_sw128(a0 + ks * 32, 16, 1024);
            uint64_t bd = tc::smem_desc_sw128(b0 + ks * 2048, 64 * 128, 1024);
            tc::mma_bf16(tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar);
    }
    tc::mbar_wait(bar, 1, abort_flag);
    tc::tc_fence_after();
    uint8_t* WU = sm + P1_WU;
    {
        // M = 64 accumulator: row m in lane (m % 16) + 32 (m / 16).  Warps w and w + 4 share lanes
        // 32 (w % 4) ..; warp w < 4 takes columns 0..127 (W), warp w + 4 columns 128..255 (U~).
        const int wq = warp & 3, half = warp >> 2;
        const int r = 16 * wq + (lane & 15);
        for (int c0 = 0; c0 < 128; c0 += 16) {
            float x[16];
            tc::tmem_ld16(tc::tmem_addr(tmem, 32 * wq, 128 * half + c0), x);
            tc::tmem_ld_wait();
            if (lane < 16) {
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    const uint4 pk = pack8(x + 8 * hc);
                    const int n = 128 * half + c0 + 8 * hc;
                    *reinterpret_cast<uint4*>(WU + tc::sw128_mnmajor(r, n, 64)) = pk;
                    if (half == 0) {
                        *reinterpret_cast<uint4*>(wsc + WS_QW + tc::sw128_kmajor(64 + r, c0 + 8 * hc, 128)) = pk;
                    } else {
                        const int nn = c0 + 8 * hc, tile = nn >> 5;
                        *reinterpret_cast<uint4*>(wsc + WS_UO + tile * WS_UO_TILE + (r * 32 + (nn & 31)) * 2) = pk;
                    }
                }
            }
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    // ======== phase F: M [W | U~]  (M = 64, N = 256, K = 64) ========
    if (tid == 0) {
        const uint32_t a0 = tc::smem_u32(sM), b0 = tc::smem_u32(WU);
        const uint32_t idesc = tc::idesc_bf16_f32(64, 256, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint64_t ad = tc::smem_desc_sw128(a0 + ks * 32, 16, 1024);
            uint64_t bd = tc::smem_desc_sw128(b0 + ks * 2048, 64 * 128, 1024);
            tc::mma_bf16(tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar);
    }
    tc::mbar_wait(bar, 0, abort_flag);
    tc::tc_fence_after();
    {
        const int wq = warp & 3, half = warp >> 2;
        const int r = 16 * wq + (lane & 15);
        for (int c0 = 0; c0 < 128; c0 += 16) {
            float x[16];
            tc::tmem_ld16(tc::tmem_addr(tmem, 32 * wq, 128 * half + c0), x);
            tc::tmem_ld_wait();
            if (lane < 16) {
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    const int n = c0 + 8 * hc;
                    float y[8];
                    if (half == 0) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = QF[r * 128 + n + e] - x[8 * hc + e];
                        *reinterpret_cast<uint4*>(wsc + WS_QW + tc::sw128_kmajor(r, n, 128)) = pack8(y);
                    } else {
                        const int tile = n >> 5;
                        *reinterpret_cast<uint4*>(wsc + WS_UO + tile * WS_UO_TILE + 4096 + (r * 32 + (n & 31)) * 2) =
                            pack8(x + 8 * hc);
                    }
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) atomicExch(&g_tc_error, 1);
    if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

// ---- kernel 2 ---------------------------------------------------------------------------------
constexpr uint32_t P2_STAGE = 58368;
constexpr uint32_t P2_QW = 0, P2_KE = 32768, P2_UO = 49152, P2_G = 57344;
constexpr uint32_t P2_LOAD_BYTES = 32768 + 16384 + WS_UO_TILE + 512;
constexpr uint32_t P2_ST = 2 * P2_STAGE;          // S^T bf16 K-major 32 rows x 128 (8 KB)
constexpr uint32_t P2_UT = P2_ST + 8192;          // U^T bf16 K-major 32 rows x 64 (4 KB)
constexpr uint32_t P2_SM = P2_UT + 4096;
constexpr uint32_t P2_BYTES = P2_SM + 256 + 1024;

__global__ void __launch_bounds__(160, 1)
ckda_tc_state(const uint8_t* __restrict__ ws, const float* __restrict__ h0,
              __nv_bfloat16* __restrict__ out, float* __restrict__ hT, int T_len, int H, int NT,
              float scale) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P2_SM);  // [2]
    uint64_t* mma1 = full + 2;
    uint64_t* mma2 = full + 3;
    uint64_t* epi1 = full + 4;
    uint64_t* epi2 = full + 5;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(full + 7);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x % kNTile, bh = blockIdx.x / kNTile;
    const int b = bh / H, h = bh % H;
    const int n0 = tile * kDVT;
    const uint8_t* wsh = ws + (size_t)bh * NT * WS_CHUNK;
    uint8_t* sST = sm + P2_ST;
    uint8_t* sUT = sm + P2_UT;

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 64);
        tc::tmem_relinquish();
    }
    if (tid == 128) {
        tc::mbar_init(&full[0], 1);
        tc::mbar_init(&full[1], 1);
        tc::mbar_init(mma1, 1);
        tc::mbar_init(mma2, 1);
        tc::mbar_init(epi1, 128);
        tc::mbar_init(epi2, 128);
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t d1 = tmem, d2 = tmem + 32;

    if (tid < 128) {
        // ---- epilogue warps: thread t owns TMEM lane t (a row of D1, a channel of D2) ----
        const int t = tid;
        float S[kDVT];
        if (h0) {
            const float4* src = reinterpret_cast<const float4*>(h0 + ((size_t)bh * kDK + t) * kDV + n0);
#pragma unroll
            for (int j = 0; j < kDVT / 4; ++j) {
                float4 x = src[j];
                S[4 * j] = x.x; S[4 * j + 1] = x.y; S[4 * j + 2] = x.z; S[4 * j + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < kDVT; ++j) S[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < kDVT; ++j) st_bf16(sST, tc::sw128_kmajor(j, t, 32), S[j]);
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::mbar_arrive(epi2);
        for (int ch = 0; ch < NT; ++ch) {
            const int st = ch & 1;
            const uint8_t* stg = sm + st * P2_STAGE;
            const int t0 = ch * kC;
            tc::mbar_wait(&full[st], (ch >> 1) & 1, abort_flag);
            tc::mbar_wait(mma1, ch & 1, abort_flag);
            tc::tc_fence_after();
            float d[32];
            tc::tmem_ld16(tc::tmem_addr(d1, 32 * warp, 0), d);
            tc::tmem_ld16(tc::tmem_addr(d1, 32 * warp, 16), d + 16);
            tc::tmem_ld_wait();
            if (t < 64) {
                const int r = t;
                const __nv_bfloat16* ol = reinterpret_cast<const __nv_bfloat16*>(stg + P2_UO + 4096) + r * 32;
                float o[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] = scale * (d[j] + __bfloat162float(ol[j]));
                if (t0 + r < T_len) {
                    uint4* dst = reinterpret_cast<uint4*>(out + (((size_t)b * T_len + t0 + r) * H + h) * kDV + n0);
#pragma unroll
                    for (int j = 0; j < 4; ++j) dst[j] = pack8(o + 8 * j);
                }
            } else {
                const int r = t - 64;
                const __nv_bfloat16* ut = reinterpret_cast<const __nv_bfloat16*>(stg + P2_UO) + r * 32;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    st_bf16(sUT, tc::sw128_kmajor(j, r, 32), __bfloat162float(ut[j]) - d[j]);
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::mbar_arrive(epi1);
            tc::mbar_wait(mma2, ch & 1, abort_flag);
            tc::tc_fence_after();
            tc::tmem_ld16(tc::tmem_addr(d2, 32 * warp, 0), d);
            tc::tmem_ld16(tc::tmem_addr(d2, 32 * warp, 16), d + 16);
            tc::tmem_ld_wait();
            const float g = reinterpret_cast<const float*>(stg + P2_G)[t];
#pragma unroll
            for (int j = 0; j < kDVT; ++j) {
                S[j] = g * S[j] + d[j];
                st_bf16(sST, tc::sw128_kmajor(j, t, 32), S[j]);
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::mbar_arrive(epi2);
        }
        if (hT) {
            float4* dst = reinterpret_cast<float4*>(hT + ((size_t)bh * kDK + t) * kDV + n0);
#pragma unroll
            for (int j = 0; j < kDVT / 4; ++j)
                dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
        }
    } else if (tid == 128) {
        // ---- control thread: stage loads (1-D bulk copies) and MMA issue ----
        auto load = [&](int c) {
            const int st = c & 1;
            uint8_t* stg = sm + st * P2_STAGE;
            const uint8_t* src = wsh + (size_t)c * WS_CHUNK;
            tc::mbar_arrive_expect_tx(&full[st], P2_LOAD_BYTES);
            tc::bulk_g2s(stg + P2_QW, src + WS_QW, 32768, &full[st]);
            tc::bulk_g2s(stg + P2_KE, src + WS_KE, 16384, &full[st]);
            tc::bulk_g2s(stg + P2_UO, src + WS_UO + tile * WS_UO_TILE, WS_UO_TILE, &full[st]);
            tc::bulk_g2s(stg + P2_G, src + WS_G, 512, &full[st]);
        };
        int loaded = 0;
        load(0);
        loaded = 1;
        const uint32_t id1 = tc::idesc_bf16_f32(128, kDVT, 0, 0);
        const uint32_t st_addr = tc::smem_u32(sST), ut_addr = tc::smem_u32(sUT);
        for (int ch = 0; ch < NT; ++ch) {
            const int st = ch & 1;
            const uint32_t stg = tc::smem_u32(sm + st * P2_STAGE);
            if (!tc::mbar_wait(epi2, ch & 1, abort_flag)) break;
            if (ch + 1 < NT) { load(ch + 1); loaded = ch + 2; }
            if (!tc::mbar_wait(&full[st], (ch >> 1) & 1, abort_flag)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint64_t ad = tc::smem_desc_sw128(stg + P2_QW + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                uint64_t bd = tc::smem_desc_sw128(st_addr + (ks >> 2) * 4096 + (ks & 3) * 32, 16, 1024);
                tc::mma_bf16(d1, ad, bd, id1, ks > 0 ? 1u : 0u);
            }
            tc::mma_commit(mma1);
            if (!tc::mbar_wait(epi1, ch & 1, abort_flag)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint64_t ad = tc::smem_desc_sw128(stg + P2_KE + ks * 32, 16, 1024);
                uint64_t bd = tc::smem_desc_sw128(ut_addr + ks * 32, 16, 1024);
                tc::mma_bf16(d2, ad, bd, id1, ks > 0 ? 1u : 0u);
            }
            tc::mma_commit(mma2);
        }
        // drain: the final epilogue arrival, then any copy still in flight
        tc::mbar_wait(epi2, NT & 1, abort_flag);
        if (*abort_flag) {
            atomicExch(&g_tc_error, 2);
            // only the latest fill of each stage can still be in flight
            for (int c = loaded > 2 ? loaded - 2 : 0; c < loaded; ++c) {
                for (uint32_t i = 0; i < tc::kSpinLimit; ++i)
                    if (tc::mbar_try_wait(&full[c & 1], (c >> 1) & 1)) break;
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 64);
    (void)lane;
}

}  // namespace

size_t chunk_tc_workspace_bytes(int B, int T_len, int H) {
    const size_t nt = (size_t)(T_len + kC - 1) / kC;
    return (size_t)B * H * nt * WS_CHUNK;
}

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const float* alpha,
                            const float* beta, const float* h0, void* out, float* hT, int B,
                            int T_len, int H, int l2norm, const RopeParams& rp, float scale,
                            long long pos_offset, void* workspace, int stages,
                            cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(ckda_tc_intra, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)P1_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ckda_tc_state, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P2_BYTES);
    if (e != cudaSuccess) return e;
    const int NT = (T_len + kC - 1) / kC;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (stages == 0) stages = 3;
    if (stages & 1) {
    ckda_tc_intra<<<(unsigned)(NT * B * H), 256, P1_BYTES, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), alpha, beta, ws, T_len, H, NT, l2norm, rp,
        pos_offset);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    }
    if (stages & 2) {
        ckda_tc_state<<<(unsigned)(kNTile * B * H), 160, P2_BYTES, stream>>>(
            ws, h0, static_cast<__nv_bfloat16*>(out), hT, T_len, H, NT, scale);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace ckda
