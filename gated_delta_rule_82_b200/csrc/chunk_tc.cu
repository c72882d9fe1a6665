// chunk_tc.cu -- chunked CKDA forward on the sm_100a tensor cores (bf16 q/k/v, dk = dv = 128,
// chunk C = 64), fp32 accumulation in Tensor Memory and an fp32 inter-chunk state.
//
// Chunk algebra (derived from the transition of the "Complex KDA" paper summary, "Background",
// A_t = (I - beta_t k_t k_t^T) Diag(alpha_t); see chunk_simt.cu for the derivation).  For a chunk
// with entering state S0 and per-channel gate products gamma_r = prod_{tau<=r} alpha_tau:
//     A_rj = beta_r k_r^T Diag(gamma_r/gamma_j) k_j (j < r),  M_rj = q_r^T Diag(gamma_r/gamma_j) k_j (j <= r)
//     T = (I + A)^-1,  W = T diag(beta) K_gamma,  U~ = T diag(beta) V
//     Q' = Q_gamma - M W,  O_loc = M U~
//     A_c = Diag(gamma_C) - K_end^T W,   B_c = K_end^T U~          (K_end,j = (gamma_C/gamma_j) k_j)
// and then, serially over chunks,
//     O = scale (Q' S0 + O_loc),      S_C = A_c S0 + B_c.
// Everything above the line is state-independent and runs chunk-parallel; the serial chain is a
// single 128 x 128 x dv product per chunk.
//
// Gates.  The sign of gamma is a parity absorbed into q and k (q' = sigma q, k' = sigma k; the
// compiled-PyTorch variant of the paper summary's "Implementation", i.e. the sign-magnitude split
// of its Proposition 2), so every ratio gamma_r/gamma_j (j <= r) is g_r / g_j with g = |gamma|, a
// product of |alpha| over (j, r].  g is formed per channel as block-local running products (16
// rows) times the totals of the earlier blocks, never as a division.  When the chunk's total
// decay g_C stays >= 2^-118 in every channel, the ratio factors exactly in floating point as
//     k'_r^T Diag(g_r / g_j) k'_j = (g_r k'_r) . (k'_j / g_j),
// with every factor inside the bf16 / fp32 exponent range (|k'/g| <= 2^118, and the products
// that are masked out, j > r, stay below 2^127), so A and M come from ONE tcgen05 product of
// L = [g k'; g q'] (128 x 128) and R = k' / g (64 x 128).  L also holds K_gamma and Q_gamma, and
// K_end = gamma_C R.  A chunk whose decay falls below 2^-118 somewhere (exact zeros, long
// stretches of tiny gates) takes an exact CUDA-core path for A and M instead, evaluating
// g_r / g_j = exp2(L_r - L_j) from an fp32 log2 prefix with non-positive exponents only.
//
// Kernel 1 (ckda_tc_intra) -- persistent, one CTA of 512 threads per SM, loops over
// (batch*head, chunk):
//   A  global loads of the next chunk-head issued together (and the one after prefetched into
//      L2); channel pass (thread per channel and 16-row block) forms the signed prefix gamma_r;
//      row pass (thread per row and two 8-channel groups, a RoPE pair) rotates and normalises q, k,
//      absorbs the signs and writes L, R, K_end with 16-byte stores.
//   B  tcgen05: [A | M] = L R^T  (M = 128, N = 64, K = 128), read back by all 16 warps.
//   C  T = (I + A)^-1 by blocked forward substitution in fp32; T' = T diag(beta) in bf16.
//   D  tcgen05: [W | U~] = T' [K_gamma | V]  (M = 64, N = 2 x 128, MN-major B).
//   F  tcgen05: M [W | U~] (M = 64) and K_end^T [W | U~] (M = 128, MN-major A).
//   G  Q', O_loc, A_c, B_c staged in shared memory and written with three bulk (TMA) stores.
// Kernel 2 (ckda_tc_state) -- one CTA per (batch*head, dv tile of 32 columns), serial over chunks:
//   a three-stage pipeline of 1-D bulk (TMA) copies of each chunk's A_c, Q', B_c and O_loc; per
//   chunk one tcgen05 product D_c = A_c S (M = 128, N = 32, K = 128) on the critical path, whose
//   epilogue adds B_c to form the fp32 master state (one row per thread, in registers) and writes
//   its bf16 copy for the next product, and one off-path product D_o = Q' S (M = 64) that becomes
//   the chunk's output.
#include "internal.cuh"
#include "tc_sm100.cuh"

namespace ckda {

namespace {

constexpr int kC = 64, kDK = 128, kDV = 128, kDVT = 32, kNTile = kDV / kDVT;

// ---- workspace image of one chunk-head (bytes) ------------------------------------------------
constexpr uint32_t WS_AC = 0;          // A_c bf16, K-major swizzled, 128 rows x 128
constexpr uint32_t WS_QP = 32768;      // Q'  bf16, K-major swizzled, 64 rows x 128
constexpr uint32_t WS_TILES = 49152;   // per dv tile t: B_c [128][32] bf16, then O_loc [64][32] bf16
constexpr uint32_t WS_TILE = 12288;
constexpr uint32_t WS_TILE_O = 8192;
constexpr uint32_t WS_CHUNK = WS_TILES + kNTile * WS_TILE;  // 98304

// ---- kernel 1 shared memory (bytes from a 1024-aligned base) ---------------------------------
constexpr uint32_t S_G = 0;          // alpha, then the signed prefix gamma (fp32 [64][128])
constexpr uint32_t S_L = 32768;      // L: rows 0..63 g k', rows 64..127 g q' (K-major, 128 rows)
constexpr uint32_t S_R = 65536;      // R = k' / g (K-major, 64 rows)
constexpr uint32_t S_V = 81920;      // V (MN-major, 64 K-rows x 128)
constexpr uint32_t S_KE = 98304;     // K_end (MN-major, 64 x 128): the MN-major A of K_end^T
constexpr uint32_t S_A = 114688;     // A fp32 [64][68]
constexpr uint32_t S_T = 132096;     // T fp32 [64][68]
constexpr uint32_t S_M = 149504;     // M bf16 K-major 64 x 64
constexpr uint32_t S_TB = 157696;    // T' bf16 K-major 64 x 64
constexpr uint32_t S_X = 165888;     // X fp32 [16][48]
constexpr uint32_t S_PT = 168960;    // partial block products fp32 [6][16][16]
constexpr uint32_t S_W = 175104;     // W MN-major 64 x 128   (exact path: log2 prefix fp32 [64][128]
constexpr uint32_t S_U = 191488;     // U~ MN-major 64 x 128   spanning S_W and S_U)
constexpr uint32_t S_SM = 207872;    // small arrays (below)
constexpr uint32_t S_BYTES = S_SM + 5120 + 1024;
constexpr int kStrideA = 68;         // fp32 row stride of A and T
// staging of the chunk's workspace image, over buffers that are dead by then
constexpr uint32_t S_OUT_AC = S_G;   // A_c image (32 KB)
constexpr uint32_t S_OUT_QP = S_R;   // Q' image (16 KB)
constexpr uint32_t S_OUT_TL = S_A;   // dv tiles (48 KB, over A, T, M and part of T')
// small arrays
constexpr uint32_t SM_P = S_SM;                  // P   fp32 [4][128]  block totals of |alpha|
constexpr uint32_t SM_PAR = S_SM + 2048;         // PAR fp32 [4][128]  block parity (+-1)
constexpr uint32_t SM_GC = S_SM + 4096;          // gamma_C fp32 [128] (signed)
constexpr uint32_t SM_B = S_SM + 4608;           // beta fp32 [64]
constexpr uint32_t SM_FLAGS = S_SM + 4864;       // int exact_path, abort, tmem slot, mbarrier

constexpr float kSafeDecay = 3.009265538105056e-36f;  // 2^-118


__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint4 pack8(const float* x) {
    return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                      pack_bf16(x[6], x[7]));
}
__device__ __forceinline__ void unpack8(uint4 v, float* x) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void st16(uint8_t* base, uint32_t off, const float* x) {
    *reinterpret_cast<uint4*>(base + off) = pack8(x);
}
__device__ __forceinline__ void ld_f8(const float* p, float* x) {
    float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ int g_tc_error;  // nonzero after a bounded wait ran out (diagnostic)

// One block-row Ib (1..3) of T = (I + A)^-1 below the diagonal, given the diagonal blocks and
// the block-rows above it:  T_{Ib,J} = -T_{Ib,Ib} sum_{K = J..Ib-1} A_{Ib,K} T_{K,J}.
// Pass 1: warp w computes one 16 x 16 x 16 product A_{Ib,K} T_{K,J} for the w-th pair J <= K < Ib;
// pass 2 sums the pairs into X; pass 3: warp J computes -T_{Ib,Ib} X_J.  Every loop is fully
// unrolled, a thread owns a 2 x 4 output tile.
template <int Ib>
__device__ __forceinline__ void t_offdiag_level(const float* sA, float* sT, float* sX, float* sPt,
                                                int tid) {
    constexpr int NP = Ib * (Ib + 1) / 2;
    const int warp = tid >> 5, lane = tid & 31;
    const int rp = lane >> 2, jq = lane & 3;
    if (warp < NP) {
        int K = 0, J = warp;
        while (J > K) { J -= K + 1; ++K; }
        const float* a0 = sA + (16 * Ib + 2 * rp) * kStrideA + 16 * K;
        const float* a1 = a0 + kStrideA;
        const float* tb = sT + (16 * K) * kStrideA + 16 * J + 4 * jq;
        float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0, y0 = x0, y1 = x0;
#pragma unroll
        for (int m = 0; m < 16; m += 2) {
            const float4 ta = *reinterpret_cast<const float4*>(tb + m * kStrideA);
            const float4 tc4 = *reinterpret_cast<const float4*>(tb + (m + 1) * kStrideA);
            const float2 aa = *reinterpret_cast<const float2*>(a0 + m);
            const float2 ab = *reinterpret_cast<const float2*>(a1 + m);
            x0.x += aa.x * ta.x; x0.y += aa.x * ta.y; x0.z += aa.x * ta.z; x0.w += aa.x * ta.w;
            y0.x += aa.y * tc4.x; y0.y += aa.y * tc4.y; y0.z += aa.y * tc4.z; y0.w += aa.y * tc4.w;
            x1.x += ab.x * ta.x; x1.y += ab.x * ta.y; x1.z += ab.x * ta.z; x1.w += ab.x * ta.w;
            y1.x += ab.y * tc4.x; y1.y += ab.y * tc4.y; y1.z += ab.y * tc4.z; y1.w += ab.y * tc4.w;
        }
        float* pt = sPt + warp * 256;
        *reinterpret_cast<float4*>(pt + (2 * rp) * 16 + 4 * jq) =
            make_float4(x0.x + y0.x, x0.y + y0.y, x0.z + y0.z, x0.w + y0.w);
        *reinterpret_cast<float4*>(pt + (2 * rp + 1) * 16 + 4 * jq) =
            make_float4(x1.x + y1.x, x1.y + y1.y, x1.z + y1.z, x1.w + y1.w);
    }
    __syncthreads();
    if (tid < 16 * 4 * Ib) {
        const int rl = tid / (4 * Ib), quad = tid % (4 * Ib);
        const int J = quad >> 2, c = 4 * (quad & 3);
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int K = 0; K < Ib; ++K) {
            if (K >= J) {
                const float4 p = *reinterpret_cast<const float4*>(sPt + (K * (K + 1) / 2 + J) * 256 + rl * 16 + c);
                x.x += p.x; x.y += p.y; x.z += p.z; x.w += p.w;
            }
        }
        *reinterpret_cast<float4*>(sX + rl * 48 + 16 * J + c) = x;
    }
    __syncthreads();
    if (warp < Ib) {
        const int J = warp;
        const float* t0r = sT + (16 * Ib + 2 * rp) * kStrideA + 16 * Ib;
        const float* t1r = t0r + kStrideA;
        const float* xb = sX + 16 * J + 4 * jq;
        float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0, y0 = x0, y1 = x0;
#pragma unroll
        for (int m = 0; m < 16; m += 2) {
            const float4 xa = *reinterpret_cast<const float4*>(xb + m * 48);
            const float4 xc = *reinterpret_cast<const float4*>(xb + (m + 1) * 48);
            const float2 aa = *reinterpret_cast<const float2*>(t0r + m);
            const float2 ab = *reinterpret_cast<const float2*>(t1r + m);
            x0.x += aa.x * xa.x; x0.y += aa.x * xa.y; x0.z += aa.x * xa.z; x0.w += aa.x * xa.w;
            y0.x += aa.y * xc.x; y0.y += aa.y * xc.y; y0.z += aa.y * xc.z; y0.w += aa.y * xc.w;
            x1.x += ab.x * xa.x; x1.y += ab.x * xa.y; x1.z += ab.x * xa.z; x1.w += ab.x * xa.w;
            y1.x += ab.y * xc.x; y1.y += ab.y * xc.y; y1.z += ab.y * xc.z; y1.w += ab.y * xc.w;
        }
        *reinterpret_cast<float4*>(sT + (16 * Ib + 2 * rp) * kStrideA + 16 * J + 4 * jq) =
            make_float4(-(x0.x + y0.x), -(x0.y + y0.y), -(x0.z + y0.z), -(x0.w + y0.w));
        *reinterpret_cast<float4*>(sT + (16 * Ib + 2 * rp + 1) * kStrideA + 16 * J + 4 * jq) =
            make_float4(-(x1.x + y1.x), -(x1.y + y1.y), -(x1.z + y1.z), -(x1.w + y1.w));
    }
    __syncthreads();
}

__global__ void __launch_bounds__(512, 1)
ckda_tc_intra(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
              const __nv_bfloat16* __restrict__ v, const float* __restrict__ alpha,
              const float* __restrict__ beta, uint8_t* __restrict__ ws, int T_len, int H, int NT,
              int total, int l2norm, RopeParams rp, long long pos_offset) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* G = reinterpret_cast<float*>(sm + S_G);
    float* gP = reinterpret_cast<float*>(sm + SM_P);
    float* gPar = reinterpret_cast<float*>(sm + SM_PAR);
    float* gGC = reinterpret_cast<float*>(sm + SM_GC);
    float* sb = reinterpret_cast<float*>(sm + SM_B);
    int* exact_path = reinterpret_cast<int*>(sm + SM_FLAGS);
    volatile int* abort_flag = exact_path + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(exact_path + 8);
    uint64_t* bar = reinterpret_cast<uint64_t*>(exact_path + 16);
    float* sA = reinterpret_cast<float*>(sm + S_A);
    float* sT = reinterpret_cast<float*>(sm + S_T);
    float* sX = reinterpret_cast<float*>(sm + S_X);
    float* sPt = reinterpret_cast<float*>(sm + S_PT);
    float* sLg = reinterpret_cast<float*>(sm + S_W);   // exact path only
    uint8_t* sM = sm + S_M;
    uint8_t* sL = sm + S_L;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t rs = (size_t)H;   // stride between tokens, in rows of [B*T*H]

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    if (tid == 32) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t phase = 0;   // completions of `bar` so far

    // persistent loop over chunk-heads ci = (batch*head) * NT + chunk
    for (int ci = blockIdx.x; ci < total; ci += gridDim.x) {
        const int ch = ci % NT, bh = ci / NT;
        const int b = bh / H, h = bh % H;
        const int t0 = ch * kC;
        const int nvalid = min(kC, T_len - t0);
        uint8_t* wsc = ws + (size_t)ci * WS_CHUNK;
        const size_t row0 = ((size_t)b * T_len + t0) * H + h;

        // ---- all global loads of this chunk-head, issued together (registers only) ----
        const int rr = tid >> 3, g = tid & 7;               // row-pass coordinates
        uint4 qkraw[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                          make_uint4(0, 0, 0, 0)};
        if (rr < nvalid) {
            const size_t o = (row0 + rr * rs) * kDK;
            qkraw[0] = *reinterpret_cast<const uint4*>(q + o + 8 * g);
            qkraw[1] = *reinterpret_cast<const uint4*>(q + o + 64 + 8 * g);
            qkraw[2] = *reinterpret_cast<const uint4*>(k + o + 8 * g);
            qkraw[3] = *reinterpret_cast<const uint4*>(k + o + 64 + 8 * g);
        }
        float4 araw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = tid + 512 * u, r = e >> 5, c4 = (e & 31) * 4;
            araw[u] = make_float4(1.f, 1.f, 1.f, 1.f);   // identity gates on padding rows
            if (r < nvalid) araw[u] = *reinterpret_cast<const float4*>(alpha + (row0 + r * rs) * kDK + c4);
        }
        uint4 vraw[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + 512 * u, r = e >> 4, n8 = (e & 15) * 8;
            vraw[u] = make_uint4(0, 0, 0, 0);
            if (r < nvalid) vraw[u] = *reinterpret_cast<const uint4*>(v + (row0 + r * rs) * kDV + n8);
        }
        const float bval = (tid < 64 && tid < nvalid) ? beta[row0 + tid * rs] : 0.f;
        // bring the next chunk-head of this CTA into L2 while this one computes: 640 lines of
        // 128 bytes (q, k, v: 2 per row; alpha: 4 per row), one or two per thread
        {
            const int nci = ci + gridDim.x;
            if (nci < total) {
                const int nch = nci % NT, nbh = nci / NT;
                const int nt0 = nch * kC, nv = min(kC, T_len - nt0);
                const size_t nrow0 = ((size_t)(nbh / H) * T_len + nt0) * H + (nbh % H);
                for (int li = tid; li < 640; li += 512) {
                    const char* p;
                    int r;
                    if (li < 384) {
                        const int which = li >> 7, rem = li & 127;
                        r = rem >> 1;
                        const __nv_bfloat16* base = which == 0 ? q : which == 1 ? k : v;
                        p = reinterpret_cast<const char*>(base + (nrow0 + r * rs) * kDK) + 128 * (rem & 1);
                    } else {
                        const int rem = li - 384;
                        r = rem >> 2;
                        p = reinterpret_cast<const char*>(alpha + (nrow0 + r * rs) * kDK) + 128 * (rem & 3);
                    }
                    if (r < nv) tc::prefetch_line_l2(p);
                }
            }
        }
        // the previous chunk-head's bulk stores must have finished reading shared memory
        if (tid == 0) tc::bulk_wait_read_all();
        __syncthreads();

        // ======== A1: alpha and V into shared memory ========
        if (tid == 0) *exact_path = 0;
        if (tid < 64) sb[tid] = bval;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = tid + 512 * u, r = e >> 5, c4 = (e & 31) * 4;
            *reinterpret_cast<float4*>(G + r * 128 + c4) = araw[u];
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + 512 * u, r = e >> 4, n8 = (e & 15) * 8;
            *reinterpret_cast<uint4*>(sm + S_V + tc::sw128_mnmajor(r, n8, 64)) = vraw[u];
        }
        __syncthreads();

        // ======== A2: channel pass -- thread (channel c, block I): signed prefix gamma ========
        const int cc = tid & 127, cI = tid >> 7;
        {
            float p = 1.f;
            bool neg = false;
#pragma unroll
            for (int rl = 0; rl < 16; ++rl) {
                const int r = 16 * cI + rl;
                const float a = G[r * 128 + cc];
                p *= fabsf(a);
                neg ^= (a < 0.f);
                G[r * 128 + cc] = neg ? -p : p;   // a signed zero keeps the parity on underflow
            }
            gP[cI * 128 + cc] = p;
            gPar[cI * 128 + cc] = neg ? -1.f : 1.f;
        }
        __syncthreads();
        {
            float pre = 1.f, all = 1.f, sC = 1.f;
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                const float P = gP[J * 128 + cc], S = gPar[J * 128 + cc];
                sC *= S;
                all *= P;
                if (J < cI) pre *= P * S;
            }
            if (pre != 1.f) {
#pragma unroll
                for (int rl = 0; rl < 16; ++rl) G[(16 * cI + rl) * 128 + cc] *= pre;
            }
            if (cI == 0) {
                gGC[cc] = sC * all;
                if (!(all >= kSafeDecay)) *exact_path = 1;
            }
        }
        __syncthreads();
        const bool exact = *exact_path != 0;

        // ======== A3: row pass -- thread (row r, 8-channel groups g and g + 8) ========
        {
            const int r = rr;
            const int cA = 8 * g, cB = 64 + 8 * g;
            float qa[8], qb[8], ka[8], kb[8];
            unpack8(qkraw[0], qa);
            unpack8(qkraw[1], qb);
            unpack8(qkraw[2], ka);
            unpack8(qkraw[3], kb);
            // row norms (the rotation preserves them): reduce over the 8 threads of the row
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                sq += qa[i] * qa[i] + qb[i] * qb[i];
                sk += ka[i] * ka[i] + kb[i] * kb[i];
            }
            sq = group_sum<8>(sq);
            sk = group_sum<8>(sk);
            if (rp.enabled) {
                const long long pos = pos_offset + t0 + r;
                if (rp.convention == 0) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {   // pairs (cA + i, cB + i), frequency 8g + i
                        float sn, cs;
                        rope_sincos(pos, rp.inv_freq[8 * g + i], &sn, &cs);
                        float x0 = qa[i], x1 = qb[i];
                        qa[i] = x0 * cs - x1 * sn; qb[i] = x1 * cs + x0 * sn;
                        x0 = ka[i]; x1 = kb[i];
                        ka[i] = x0 * cs - x1 * sn; kb[i] = x1 * cs + x0 * sn;
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < 4; ++m) {   // pairs (c, c + 1) inside each 8-channel group
                        float sn, cs;
                        rope_sincos(pos, rp.inv_freq[4 * g + m], &sn, &cs);
                        float x0 = qa[2 * m], x1 = qa[2 * m + 1];
                        qa[2 * m] = x0 * cs - x1 * sn; qa[2 * m + 1] = x1 * cs + x0 * sn;
                        x0 = ka[2 * m]; x1 = ka[2 * m + 1];
                        ka[2 * m] = x0 * cs - x1 * sn; ka[2 * m + 1] = x1 * cs + x0 * sn;
                        rope_sincos(pos, rp.inv_freq[32 + 4 * g + m], &sn, &cs);
                        x0 = qb[2 * m]; x1 = qb[2 * m + 1];
                        qb[2 * m] = x0 * cs - x1 * sn; qb[2 * m + 1] = x1 * cs + x0 * sn;
                        x0 = kb[2 * m]; x1 = kb[2 * m + 1];
                        kb[2 * m] = x0 * cs - x1 * sn; kb[2 * m + 1] = x1 * cs + x0 * sn;
                    }
                }
            }
            const float fq = l2norm ? rsqrtf(sq + kL2Eps) : 1.f;
            const float fk = l2norm ? rsqrtf(sk + kL2Eps) : 1.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int c0 = hh ? cB : cA;
                const float* qx = hh ? qb : qa;
                const float* kx = hh ? kb : ka;
                float gm[8], kp[8], qp[8], t8[8];
                ld_f8(G + r * 128 + c0, gm);   // gamma_r: |gamma| with the parity as its sign
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float sg = signbit(gm[i]) ? -1.f : 1.f;
                    kp[i] = kx[i] * fk * sg;   // k'
                    qp[i] = qx[i] * fq * sg;   // q'
                    gm[i] = fabsf(gm[i]);      // g
                }
                if (!exact) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) t8[i] = kp[i] * gm[i];
                    st16(sL, tc::sw128_kmajor(r, c0, 128), t8);          // g k'  (= K_gamma)
#pragma unroll
                    for (int i = 0; i < 8; ++i) t8[i] = qp[i] * gm[i];
                    st16(sL, tc::sw128_kmajor(64 + r, c0, 128), t8);     // g q'  (= Q_gamma)
                    float ke[8];
                    ld_f8(gGC + c0, ke);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        t8[i] = kp[i] * __frcp_rn(gm[i]);                // k' / g
                        ke[i] *= t8[i];                                  // gamma_C k' / g
                    }
                    st16(sm + S_R, tc::sw128_kmajor(r, c0, 64), t8);
                    st16(sm + S_KE, tc::sw128_mnmajor(r, c0, 64), ke);   // K_end
                } else {
                    // exact path: unscaled k', q' for the CUDA-core A and M
                    st16(sL, tc::sw128_kmajor(r, c0, 128), kp);
                    st16(sL, tc::sw128_kmajor(64 + r, c0, 128), qp);
                }
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();

        if (!exact) {
            // ======== B: [A | M] = L R^T on the tensor cores (M = 128, N = 64, K = 128) ========
            if (tid == 0) {
                const uint32_t l0 = tc::smem_u32(sL), r0a = tc::smem_u32(sm + S_R);
                const uint32_t idesc = tc::idesc_bf16_f32(128, 64, 0, 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad = tc::smem_desc_sw128(l0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                    const uint64_t bd = tc::smem_desc_sw128(r0a + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                    tc::mma_bf16(tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
                }
                tc::mma_commit(bar);
            }
            tc::mbar_wait(bar, phase & 1, abort_flag);
            ++phase;
            tc::tc_fence_after();
            {
                // TMEM lanes 0..63: rows of A (k rows); lanes 64..127: rows of M (q rows).
                // Warp w: lanes 32 (w % 4) .., columns 16 (w / 4) ..
                const int quarter = warp & 3, c0 = 16 * (warp >> 2);
                float x[16];
                tc::tmem_ld16_sync(tc::tmem_addr(tmem, 32 * quarter, c0), x);
                const int r = 32 * (quarter & 1) + lane;
                if (quarter < 2) {
                    const float br = sb[r];
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] = (c0 + i) < r ? br * x[i] : 0.f;
#pragma unroll
                    for (int i = 0; i < 16; i += 4)
                        *reinterpret_cast<float4*>(sA + r * kStrideA + c0 + i) =
                            make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] = (c0 + i) <= r ? x[i] : 0.f;
                    st16(sM, tc::sw128_kmajor(r, c0, 64), x);
                    st16(sM, tc::sw128_kmajor(r, c0 + 8, 64), x + 8);
                }
            }
        } else {
            // ======== exact path for A and M (chunks whose decay leaves the bf16 range) ========
            // log2 prefix L_r = sum_{tau <= r} log2 max(|alpha_tau|, FLT_MIN), straight from alpha
            if (tid < 128) {
                float L = 0.f;
                for (int r = 0; r < 64; ++r) {
                    const float a = r < nvalid ? alpha[(row0 + r * rs) * kDK + tid] : 1.f;
                    L += log2f(fmaxf(fabsf(a), 1.17549435e-38f));
                    sLg[r * 128 + tid] = L;
                }
            }
            __syncthreads();
            for (int pr = tid; pr < 64 * 64; pr += 512) {
                const int r = pr >> 6, j = pr & 63;
                float accA = 0.f, accM = 0.f;
                if (j <= r) {
                    for (int c = 0; c < kDK; ++c) {
                        const float e = exp2f(sLg[r * 128 + c] - sLg[j * 128 + c]);
                        const float kj = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sL + tc::sw128_kmajor(j, c, 128))) * e;
                        accA += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sL + tc::sw128_kmajor(r, c, 128))) * kj;
                        accM += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sL + tc::sw128_kmajor(64 + r, c, 128))) * kj;
                    }
                }
                sA[r * kStrideA + j] = j < r ? sb[r] * accA : 0.f;
                *reinterpret_cast<__nv_bfloat16*>(sM + tc::sw128_kmajor(r, j, 64)) = __float2bfloat16_rn(accM);
            }
            __syncthreads();
            // rescale L to (g k', g q') with g = exp2(L_r) and form K_end = sigma_C exp2(L_C - L_j) k'
            for (int e = tid; e < 64 * 128; e += 512) {
                const int r = e >> 7, c = e & 127;
                const float gr = exp2f(sLg[r * 128 + c]);
                __nv_bfloat16* kr = reinterpret_cast<__nv_bfloat16*>(sL + tc::sw128_kmajor(r, c, 128));
                __nv_bfloat16* qr = reinterpret_cast<__nv_bfloat16*>(sL + tc::sw128_kmajor(64 + r, c, 128));
                const float kv = __bfloat162float(*kr), qv = __bfloat162float(*qr);
                const float sC = signbit(gGC[c]) ? -1.f : 1.f;
                *reinterpret_cast<__nv_bfloat16*>(sm + S_KE + tc::sw128_mnmajor(r, c, 64)) =
                    __float2bfloat16_rn(sC * exp2f(sLg[63 * 128 + c] - sLg[r * 128 + c]) * kv);
                *kr = __float2bfloat16_rn(gr * kv);
                *qr = __float2bfloat16_rn(gr * qv);
            }
        }
        tc::tc_fence_before();
        __syncthreads();

        // ======== C: T = (I + A)^-1 (fp32), T' = T diag(beta) (bf16) ========
        for (int e = tid; e < 64 * 64; e += 512) {
            const int r = e >> 6, j = e & 63;
            if ((j >> 4) > (r >> 4)) sT[r * kStrideA + j] = 0.f;
        }
        if (warp < 4 && lane < 16) {
            const int J = warp, l = lane, base = 16 * J;
            float tcol[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int m = 0; m < 16; m += 2) {
                    if (m < i) a0 += sA[(base + i) * kStrideA + base + m] * tcol[m];
                    if (m + 1 < i) a1 += sA[(base + i) * kStrideA + base + m + 1] * tcol[m + 1];
                }
                tcol[i] = i < l ? 0.f : (i == l ? 1.f : -(a0 + a1));
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) sT[(base + i) * kStrideA + base + l] = tcol[i];
        }
        __syncthreads();
        t_offdiag_level<1>(sA, sT, sX, sPt, tid);
        t_offdiag_level<2>(sA, sT, sX, sPt, tid);
        t_offdiag_level<3>(sA, sT, sX, sPt, tid);
        for (int e = tid; e < 64 * 8; e += 512) {
            const int r = e >> 3, j0 = (e & 7) * 8;
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = sT[r * kStrideA + j0 + i] * sb[j0 + i];
            st16(sm + S_TB, tc::sw128_kmajor(r, j0, 64), y);
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();

        // ======== D: W = T' K_gamma, U~ = T' V  (M = 64, N = 128 each, K = 64) ========
        // K_gamma is rows 0..63 of L, read as an MN-major operand: 64-column blocks 16 KB apart.
        if (tid == 0) {
            const uint32_t a0 = tc::smem_u32(sm + S_TB);
            const uint32_t kg = tc::smem_u32(sL), vv = tc::smem_u32(sm + S_V);
            const uint32_t idesc = tc::idesc_bf16_f32(64, 128, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = tc::smem_desc_sw128(a0 + ks * 32, 16, 1024);
                tc::mma_bf16(tmem, ad, tc::smem_desc_sw128(kg + ks * 2048, 16384, 1024), idesc, ks > 0);
                tc::mma_bf16(tmem + 128, ad, tc::smem_desc_sw128(vv + ks * 2048, 8192, 1024), idesc, ks > 0);
            }
            tc::mma_commit(bar);
        }
        tc::mbar_wait(bar, phase & 1, abort_flag);
        ++phase;
        tc::tc_fence_after();
        {
            // warp w: rows 16 (w % 4) + lane (lane < 16); 64-column slice w / 4:
            // slices 0, 1 -> W columns 0..127, slices 2, 3 -> U~ columns 0..127
            const int quarter = warp & 3, slice = warp >> 2;
            const int r = 16 * quarter + (lane & 15);
            uint8_t* dst = sm + (slice < 2 ? S_W : S_U);
            const int n0 = 64 * (slice & 1);
            float x[64];
            tc::tmem_ld64_sync(tc::tmem_addr(tmem, 32 * quarter, 64 * slice), x);
            if (lane < 16) {
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 8) st16(dst, tc::sw128_mnmajor(r, n0 + c0, 64), x + c0);
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();

        // ======== F: M [W | U~] (M = 64) and K_end^T [W | U~] (M = 128, MN-major A) ========
        if (tid == 0) {
            const uint32_t am = tc::smem_u32(sm + S_M), ke = tc::smem_u32(sm + S_KE);
            const uint32_t w0 = tc::smem_u32(sm + S_W), u0 = tc::smem_u32(sm + S_U);
            const uint32_t id64 = tc::idesc_bf16_f32(64, 128, 0, 1);
            const uint32_t id128 = tc::idesc_bf16_f32(128, 128, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t bw = tc::smem_desc_sw128(w0 + ks * 2048, 8192, 1024);
                const uint64_t bu = tc::smem_desc_sw128(u0 + ks * 2048, 8192, 1024);
                const uint64_t adm = tc::smem_desc_sw128(am + ks * 32, 16, 1024);
                const uint64_t ade = tc::smem_desc_sw128(ke + ks * 2048, 8192, 1024);
                tc::mma_bf16(tmem, adm, bw, id64, ks > 0);
                tc::mma_bf16(tmem + 128, adm, bu, id64, ks > 0);
                tc::mma_bf16(tmem + 256, ade, bw, id128, ks > 0);
                tc::mma_bf16(tmem + 384, ade, bu, id128, ks > 0);
            }
            tc::mma_commit(bar);
        }
        tc::mbar_wait(bar, phase & 1, abort_flag);
        ++phase;
        tc::tc_fence_after();
        // ======== G: results into shared staging images, then three bulk stores ========
        {
            const int quarter = warp & 3, slice = warp >> 2;
            // (1) M = 64 products: rows 16 quarter + lane; slices 0, 1 -> Q', 2, 3 -> O_loc
            {
                const int r = 16 * quarter + (lane & 15);
                const int n0 = 64 * (slice & 1);
                float x[64];
                tc::tmem_ld64_sync(tc::tmem_addr(tmem, 32 * quarter, 64 * slice), x);
                if (lane < 16) {
#pragma unroll
                    for (int c0 = 0; c0 < 64; c0 += 8) {
                        const int n = n0 + c0;
                        if (slice < 2) {
                            float qg[8];
                            unpack8(*reinterpret_cast<const uint4*>(sL + tc::sw128_kmajor(64 + r, n, 128)), qg);
#pragma unroll
                            for (int i = 0; i < 8; ++i) qg[i] -= x[c0 + i];
                            st16(sm + S_OUT_QP, tc::sw128_kmajor(r, n, 64), qg);
                        } else {
                            st16(sm + S_OUT_TL, (n >> 5) * WS_TILE + WS_TILE_O + (r * 32 + (n & 31)) * 2, x + c0);
                        }
                    }
                }
            }
            // (2) M = 128 products: row c' = 32 quarter + lane; slices 0, 1 -> A_c, 2, 3 -> B_c
            {
                const int cr = 32 * quarter + lane;
                const int n0 = 64 * (slice & 1);
                const float gc = gGC[cr];
                float x[64];
                tc::tmem_ld64_sync(tc::tmem_addr(tmem, 32 * quarter, 256 + 64 * slice), x);
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 8) {
                    const int n = n0 + c0;
                    if (slice < 2) {
                        float y[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) y[i] = (n + i == cr ? gc : 0.f) - x[c0 + i];
                        st16(sm + S_OUT_AC, tc::sw128_kmajor(cr, n, 128), y);
                    } else {
                        st16(sm + S_OUT_TL, (n >> 5) * WS_TILE + (cr * 32 + (n & 31)) * 2, x + c0);
                    }
                }
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
        if (tid == 0) {
            tc::bulk_s2g(wsc + WS_AC, sm + S_OUT_AC, 32768);
            tc::bulk_s2g(wsc + WS_QP, sm + S_OUT_QP, 16384);
            tc::bulk_s2g(wsc + WS_TILES, sm + S_OUT_TL, kNTile * WS_TILE);
            tc::bulk_commit();
        }
    }
    if (tid == 0) tc::bulk_wait_all();
    tc::tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) atomicExch(&g_tc_error, 1);
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ---- kernel 2: the serial state pass ------------------------------------------------------------
constexpr int kStages = 3;
constexpr uint32_t P2_STAGE = 61440;                    // A_c 32 KB, Q' 16 KB, B_c 8 KB, O_loc 4 KB
constexpr uint32_t P2_AC = 0, P2_QP = 32768, P2_BC = 49152, P2_OL = 57344;
constexpr uint32_t P2_LOAD_BYTES = 32768 + 16384 + WS_TILE;
constexpr uint32_t P2_ST = kStages * P2_STAGE;          // S operand bf16, K-major 32 rows x 128
constexpr uint32_t P2_SM = P2_ST + 8192;
constexpr uint32_t P2_BYTES = P2_SM + 256 + 1024;

__global__ void __launch_bounds__(160, 1)
ckda_tc_state(const uint8_t* __restrict__ ws, const float* __restrict__ h0,
              __nv_bfloat16* __restrict__ out, float* __restrict__ hT, int T_len, int H, int NT,
              float scale) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P2_SM);  // [3]
    uint64_t* empty = full + 3;                                // [3]
    uint64_t* mma_c = full + 6;
    uint64_t* mma_o = full + 7;
    uint64_t* epi = full + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + 9);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(full + 10);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x % kNTile, bh = blockIdx.x / kNTile;
    const int b = bh / H, h = bh % H;
    const int n0 = tile * kDVT;
    const uint8_t* wsh = ws + (size_t)bh * NT * WS_CHUNK;
    uint8_t* sST = sm + P2_ST;

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 128);
        tc::tmem_relinquish();
    }
    if (tid == 128) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 128);
        }
        tc::mbar_init(mma_c, 1);
        tc::mbar_init(mma_o, 1);
        tc::mbar_init(epi, 128);
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t dc = tmem;                 // D_c: 128 lanes x 32 columns
    const uint32_t dob = tmem + 32;           // D_o: two buffers of 32 columns (M = 64 layout)

    if (tid < 128) {
        // ---- epilogue: thread t owns state row t (TMEM lane t of D_c) ----
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
        for (int j = 0; j < kDVT; ++j)
            *reinterpret_cast<__nv_bfloat16*>(sST + tc::sw128_kmajor(j, t, 32)) = __float2bfloat16_rn(S[j]);
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::mbar_arrive(epi);
        for (int ch = 0; ch < NT; ++ch) {
            const int st = ch % kStages;
            const uint8_t* stg = sm + st * P2_STAGE;
            // chain: S = D_c + B_c
            tc::mbar_wait(mma_c, ch & 1, abort_flag);
            tc::mbar_wait(&full[st], (ch / kStages) & 1, abort_flag);
            tc::tc_fence_after();
            float d[32];
            tc::tmem_ld32_sync(tc::tmem_addr(dc, 32 * warp, 0), d);
            const uint4* bc = reinterpret_cast<const uint4*>(stg + P2_BC + t * 64);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float y[8];
                unpack8(bc[j], y);
#pragma unroll
                for (int i = 0; i < 8; ++i) S[8 * j + i] = d[8 * j + i] + y[i];
            }
#pragma unroll
            for (int j = 0; j < kDVT; ++j)
                *reinterpret_cast<__nv_bfloat16*>(sST + tc::sw128_kmajor(j, t, 32)) = __float2bfloat16_rn(S[j]);
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::mbar_arrive(epi);
            // output (off the critical path): O = scale (D_o + O_loc), rows in the M = 64 layout
            tc::mbar_wait(mma_o, ch & 1, abort_flag);
            tc::tc_fence_after();
            tc::tmem_ld32_sync(tc::tmem_addr(dob + 32 * (ch & 1), 32 * warp, 0), d);
            if (lane < 16) {
                const int r = 16 * warp + lane;
                const int t0 = ch * kC;
                if (t0 + r < T_len) {
                    const uint4* ol = reinterpret_cast<const uint4*>(stg + P2_OL + r * 64);
                    uint4* dst = reinterpret_cast<uint4*>(out + (((size_t)b * T_len + t0 + r) * H + h) * kDV + n0);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        float y[8];
                        unpack8(ol[j], y);
#pragma unroll
                        for (int i = 0; i < 8; ++i) y[i] = scale * (d[8 * j + i] + y[i]);
                        dst[j] = pack8(y);
                    }
                }
            }
            tc::tc_fence_before();
            tc::mbar_arrive(&empty[st]);
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
            const int st = c % kStages;
            uint8_t* stg = sm + st * P2_STAGE;
            const uint8_t* src = wsh + (size_t)c * WS_CHUNK;
            tc::mbar_arrive_expect_tx(&full[st], P2_LOAD_BYTES);
            tc::bulk_g2s(stg + P2_AC, src + WS_AC, 32768, &full[st]);
            tc::bulk_g2s(stg + P2_QP, src + WS_QP, 16384, &full[st]);
            tc::bulk_g2s(stg + P2_BC, src + WS_TILES + tile * WS_TILE, WS_TILE, &full[st]);
        };
        int issued = 0;
        for (; issued < kStages && issued < NT; ++issued) load(issued);
        const uint32_t idc = tc::idesc_bf16_f32(128, kDVT, 0, 0);
        const uint32_t ido = tc::idesc_bf16_f32(64, kDVT, 0, 0);
        const uint32_t s_addr = tc::smem_u32(sST);
        for (int ch = 0; ch < NT; ++ch) {
            const int st = ch % kStages;
            const uint32_t stg = tc::smem_u32(sm + st * P2_STAGE);
            if (!tc::mbar_wait(epi, ch & 1, abort_flag)) break;            // S operand ready
            if (!tc::mbar_wait(&full[st], (ch / kStages) & 1, abort_flag)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t bd = tc::smem_desc_sw128(s_addr + (ks >> 2) * 4096 + (ks & 3) * 32, 16, 1024);
                const uint64_t ad = tc::smem_desc_sw128(stg + P2_AC + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                tc::mma_bf16(dc, ad, bd, idc, ks > 0 ? 1u : 0u);
            }
            tc::mma_commit(mma_c);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t bd = tc::smem_desc_sw128(s_addr + (ks >> 2) * 4096 + (ks & 3) * 32, 16, 1024);
                const uint64_t ad = tc::smem_desc_sw128(stg + P2_QP + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                tc::mma_bf16(dob + 32 * (ch & 1), ad, bd, ido, ks > 0 ? 1u : 0u);
            }
            tc::mma_commit(mma_o);
            // refill the stage of chunk ch - 1 once its epilogue has consumed it
            if (ch >= 1 && issued < NT) {
                const int prev = ch - 1;
                if (!tc::mbar_wait(&empty[prev % kStages], (prev / kStages) & 1, abort_flag)) break;
                load(issued);
                ++issued;
            }
        }
        // drain: the last output epilogue, then any copy still in flight
        if (NT > 0) tc::mbar_wait(&empty[(NT - 1) % kStages], ((NT - 1) / kStages) & 1, abort_flag);
        if (*abort_flag) {
            atomicExch(&g_tc_error, 2);
            for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
                for (uint32_t i = 0; i < tc::kSpinLimit; ++i)
                    if (tc::mbar_try_wait(&full[c % kStages], (c / kStages) & 1)) break;
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 128);
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
                                         (int)S_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ckda_tc_state, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P2_BYTES);
    if (e != cudaSuccess) return e;
    const int NT = (T_len + kC - 1) / kC;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (stages == 0) stages = 3;
    if (stages & 1) {
        int dev = 0, nsm = 148;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        const int total = NT * B * H;
        const int grid = total < nsm ? total : nsm;
        ckda_tc_intra<<<(unsigned)grid, 512, S_BYTES, stream>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
            static_cast<const __nv_bfloat16*>(v), alpha, beta, ws, T_len, H, NT, total, l2norm, rp,
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
