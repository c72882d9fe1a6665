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
// of its Proposition 2), so every ratio gamma_r/gamma_j (j <= r) is a product of |alpha| over
// (j, r].  Those products are formed block-locally on 16-row blocks and never by dividing
// chunk-long products:
//   fb_r  = prod |alpha| from the block start to r (inclusive)        <= 1
//   bb_j  = prod |alpha| over (j, block end]                           <= 1
//   P_I   = block total;  off-diagonal block (I > J):  ratio = fb_r * prod_{J<J'<I} P_J' * bb_j
// so both GEMM operands of an off-diagonal block lie in [0, 1].  Inside a diagonal block the ratio
// is fb_r / fb_j, bounded by 2^60 while the block total is >= 2^-60 (gates averaging |alpha| >=
// 2^-3.75); a block below that (exact zeros, very strong decay) is recomputed exactly on CUDA
// cores with running products from the inputs in global memory.
//
// Kernel 1 (ckda_tc_intra) -- one CTA of 512 threads per (batch*head, chunk):
//   A  alpha staged in shared memory; channel pass (thread per channel and 16-row block) forms the
//      signed block prefix fb (sign = block-local parity), the suffix bb and the block totals;
//      row pass (thread per row and 16 channels: a RoPE pair of 8-channel groups) loads q, k with
//      16-byte loads, rotates, normalises, absorbs the signs and writes every operand tile with
//      16-byte stores: L (k'fb | q'fb per block), the B tiles, K_gamma, K_end, Q_gamma, V.
//   B  tcgen05: A and M block-rows (M = 64, K = 128) into TMEM; read back by 8 warps.
//   C  T = (I + A)^-1 by blocked forward substitution in fp32; T' = T diag(beta) in bf16.
//   D  tcgen05: [W | U~] = T' [K_gamma | V]  (M = 64, N = 2 x 128, MN-major B).
//   F  tcgen05: M [W | U~] (M = 64) and K_end^T [W | U~] (M = 128, MN-major A).
//   G  write Q', O_loc, A_c, B_c as UMMA-ready images / dv tiles of the workspace.
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
constexpr uint32_t S_FB = 0;         // alpha, then signed fb (fp32 [64][128]); later A, T, M, T', X
constexpr uint32_t S_BB = 32768;     // bb (fp32 [64][128])
constexpr uint32_t S_L = 65536;      // L tile (K-major, 128 rows); later W and U~ tiles (MN-major)
constexpr uint32_t S_B = 98304;      // B tiles (16 + 32 + 48 + 64 rows); later fallback scratch
constexpr uint32_t S_KG = 139264;    // K_gamma (MN-major, 64 K-rows x 128)
constexpr uint32_t S_V = 155648;     // V (MN-major, 64 x 128)
constexpr uint32_t S_KE = 172032;    // K_end (MN-major, 64 x 128): the MN-major A of K_end^T
constexpr uint32_t S_QG = 188416;    // Q_gamma (K-major, 64 rows x 128)
constexpr uint32_t S_SM = 204800;    // small arrays (below)
constexpr uint32_t S_BYTES = S_SM + 13312 + 1024;

constexpr int kStrideA = 68;                     // fp32 row stride of A and T
constexpr uint32_t S_A = 0;                      // A  fp32 [64][68]
constexpr uint32_t S_T = 17408;                  // T  fp32 [64][68]
constexpr uint32_t S_M = 35840;                  // M  bf16 K-major 64 x 64
constexpr uint32_t S_TB = 44032;                 // T' bf16 K-major 64 x 64
constexpr uint32_t S_X = 52224;                  // X  fp32 [16][48]
constexpr uint32_t S_PT = 55296;                 // partial block products fp32 [6][16][16]
constexpr uint32_t S_W = S_L;                    // W  MN-major 64 x 128
constexpr uint32_t S_U = S_L + 16384;            // U~ MN-major 64 x 128
constexpr uint32_t S_FQ = S_B;                   // fallback q' fp32 [16][128]
constexpr uint32_t S_FK = S_B + 8192;            // fallback k' fp32 [16][128]
constexpr uint32_t S_OUT = 0;                    // staging of the chunk's workspace image (96 KB)
// small arrays
constexpr uint32_t SM_P = S_SM;                  // P    fp32 [4][128]  block totals of |alpha|
constexpr uint32_t SM_PAR = S_SM + 2048;         // PAR  fp32 [4][128]  block parity (+-1)
constexpr uint32_t SM_PRE = S_SM + 4096;         // PRE  fp32 [4][128]  prod_{J<I} P_J
constexpr uint32_t SM_KEF = S_SM + 6144;         // KEF  fp32 [4][128]  sigma_C prod_{J>I} P_J
constexpr uint32_t SM_OFF2 = S_SM + 8192;        // OFF2 fp32 [4][128]  P_{I+1}
constexpr uint32_t SM_OFF3 = S_SM + 10240;       // OFF3 fp32 [4][128]  P_{I+1} P_{I+2}
constexpr uint32_t SM_GC = S_SM + 12288;         // gamma_C fp32 [128]
constexpr uint32_t SM_B = S_SM + 12800;          // beta fp32 [64]
constexpr uint32_t SM_FLAGS = S_SM + 13056;      // int unsafe[4], abort, tmem slot, mbarrier

__host__ __device__ constexpr uint32_t btile_off(int I) { return I == 0 ? 0u : I == 1 ? 4096u : I == 2 ? 12288u : 24576u; }
__host__ __device__ constexpr uint32_t amcol(int I) { return I == 0 ? 0u : I == 1 ? 16u : I == 2 ? 48u : 96u; }

constexpr float kDiagSafe = 8.673617379884035e-19f;  // 2^-60

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

// Recompute one row of q' and k' (rotation, L2 norm, chunk-local sign parity) straight from the
// inputs; used only by the exact fallback of a collapsed diagonal block.  One warp per row.
__device__ void fallback_row(const __nv_bfloat16* q, const __nv_bfloat16* k, const float* alpha,
                             size_t row0, size_t rs, int r, int lane, const RopeParams& rp,
                             long long pos, int l2norm, float* fq, float* fk) {
    float qv[4], kv[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int c = lane + 32 * m;
        qv[m] = __bfloat162float(q[(row0 + (size_t)r * rs) * kDK + c]);
        kv[m] = __bfloat162float(k[(row0 + (size_t)r * rs) * kDK + c]);
    }
    if (rp.enabled) {
        float qn[4], kn[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int c = lane + 32 * m;
            int i;
            bool first;
            float qp, kp;
            if (rp.convention == 0) {   // partner c ^ 64: same lane, m ^ 2
                i = c & 63; first = c < 64; qp = qv[m ^ 2]; kp = kv[m ^ 2];
            } else {                    // partner c ^ 1: neighbouring lane
                i = c >> 1; first = (c & 1) == 0;
                qp = __shfl_xor_sync(0xffffffffu, qv[m], 1);
                kp = __shfl_xor_sync(0xffffffffu, kv[m], 1);
            }
            float sn, cs;
            rope_sincos(pos, rp.inv_freq[i], &sn, &cs);
            qn[m] = first ? qv[m] * cs - qp * sn : qv[m] * cs + qp * sn;
            kn[m] = first ? kv[m] * cs - kp * sn : kv[m] * cs + kp * sn;
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) { qv[m] = qn[m]; kv[m] = kn[m]; }
    }
    if (l2norm) {
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) { a += qv[m] * qv[m]; b += kv[m] * kv[m]; }
        a = rsqrtf(warp_sum(a) + kL2Eps);
        b = rsqrtf(warp_sum(b) + kL2Eps);
#pragma unroll
        for (int m = 0; m < 4; ++m) { qv[m] *= a; kv[m] *= b; }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int c = lane + 32 * m;
        float sg = 1.f;
        for (int tau = 0; tau <= r; ++tau)
            if (alpha[(row0 + (size_t)tau * rs) * kDK + c] < 0.f) sg = -sg;
        fq[c] = sg * qv[m];
        fk[c] = sg * kv[m];
    }
}


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
    float* FB = reinterpret_cast<float*>(sm + S_FB);
    float* BB = reinterpret_cast<float*>(sm + S_BB);
    float* gP = reinterpret_cast<float*>(sm + SM_P);
    float* gPar = reinterpret_cast<float*>(sm + SM_PAR);
    float* gPre = reinterpret_cast<float*>(sm + SM_PRE);
    float* gKef = reinterpret_cast<float*>(sm + SM_KEF);
    float* gOff2 = reinterpret_cast<float*>(sm + SM_OFF2);
    float* gOff3 = reinterpret_cast<float*>(sm + SM_OFF3);
    float* gGC = reinterpret_cast<float*>(sm + SM_GC);
    float* sb = reinterpret_cast<float*>(sm + SM_B);
    int* unsafe = reinterpret_cast<int*>(sm + SM_FLAGS);
    volatile int* abort_flag = unsafe + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(unsafe + 8);
    uint64_t* bar = reinterpret_cast<uint64_t*>(unsafe + 16);
    float* sA = reinterpret_cast<float*>(sm + S_A);
    float* sT = reinterpret_cast<float*>(sm + S_T);
    float* sX = reinterpret_cast<float*>(sm + S_X);
    uint8_t* sM = sm + S_M;
    uint8_t* out = sm + S_OUT;

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
        // the previous chunk-head's bulk store must have finished reading shared memory
        if (tid == 0) tc::bulk_wait_read_all();
        __syncthreads();

        // ======== A1: alpha and V into shared memory ========
        if (tid < 4) unsafe[tid] = 0;
        if (tid < 64) sb[tid] = bval;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = tid + 512 * u, r = e >> 5, c4 = (e & 31) * 4;
            *reinterpret_cast<float4*>(FB + r * 128 + c4) = araw[u];
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + 512 * u, r = e >> 4, n8 = (e & 15) * 8;
            *reinterpret_cast<uint4*>(sm + S_V + tc::sw128_mnmajor(r, n8, 64)) = vraw[u];
        }
        __syncthreads();

        // ======== A2: channel pass -- thread (channel c, block I) ========
        const int cc = tid & 127, cI = tid >> 7;
        {
            float bbv = 1.f;
#pragma unroll
            for (int rl = 15; rl >= 0; --rl) {
                const int r = 16 * cI + rl;
                BB[r * 128 + cc] = bbv;
                bbv *= fabsf(FB[r * 128 + cc]);
            }
            float p = 1.f;
            bool neg = false;
#pragma unroll
            for (int rl = 0; rl < 16; ++rl) {
                const int r = 16 * cI + rl;
                const float a = FB[r * 128 + cc];
                p *= fabsf(a);
                neg ^= (a < 0.f);
                FB[r * 128 + cc] = neg ? -p : p;   // a signed zero keeps the parity on underflow
            }
            gP[cI * 128 + cc] = p;
            gPar[cI * 128 + cc] = neg ? -1.f : 1.f;
            if (!(p >= kDiagSafe)) unsafe[cI] = 1;
        }
        __syncthreads();
        // A2b: per-(block, channel) factors; the parity before the block goes into FB's sign
        {
            float spre = 1.f, pre = 1.f, suf = 1.f, sC = 1.f, all = 1.f;
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                const float P = gP[J * 128 + cc], S = gPar[J * 128 + cc];
                sC *= S;
                all *= P;
                if (J < cI) { spre *= S; pre *= P; }
                if (J > cI) suf *= P;
            }
            if (spre < 0.f) {
#pragma unroll
                for (int rl = 0; rl < 16; ++rl) FB[(16 * cI + rl) * 128 + cc] = -FB[(16 * cI + rl) * 128 + cc];
            }
            gPre[cI * 128 + cc] = pre;
            gKef[cI * 128 + cc] = sC * suf;
            gOff2[cI * 128 + cc] = cI + 1 < 4 ? gP[(cI + 1) * 128 + cc] : 0.f;
            gOff3[cI * 128 + cc] = cI + 2 < 4 ? gP[(cI + 1) * 128 + cc] * gP[(cI + 2) * 128 + cc] : 0.f;
            if (cI == 0) gGC[cc] = sC * all;   // gamma_C (signed)
        }
        __syncthreads();

        // ======== A3: row pass -- thread (row r, 8-channel groups g and g + 8) ========
        {
            const int r = rr, I = r >> 4, rl = r & 15;
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
            const bool diag_ok = !unsafe[I];
            // A3a: the operands of the A / M products (L and B tiles)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int c0 = hh ? cB : cA;
                const float* qx = hh ? qb : qa;
                const float* kx = hh ? kb : ka;
                float fb[8], kp[8], qp[8], acc[8], t8[8];
                ld_f8(FB + r * 128 + c0, fb);   // |fb| with the full-chunk parity as its sign
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float sg = signbit(fb[i]) ? -1.f : 1.f;
                    kp[i] = kx[i] * fk * sg;
                    qp[i] = qx[i] * fq * sg;
                    fb[i] = fabsf(fb[i]);
                }
                // L tile: k' fb and q' fb
#pragma unroll
                for (int i = 0; i < 8; ++i) t8[i] = kp[i] * fb[i];
                st16(sm + S_L, tc::sw128_kmajor(32 * I + rl, c0, 128), t8);
#pragma unroll
                for (int i = 0; i < 8; ++i) t8[i] = qp[i] * fb[i];
                st16(sm + S_L, tc::sw128_kmajor(32 * I + 16 + rl, c0, 128), t8);
                // right operand of the diagonal block: k' / fb
#pragma unroll
                for (int i = 0; i < 8; ++i) t8[i] = diag_ok ? kp[i] * __frcp_rn(fb[i]) : 0.f;
                st16(sm + S_B + btile_off(I), tc::sw128_kmajor(r, c0, 16 * (I + 1)), t8);
                // off-diagonal right operands k' bb prod_{I<J<I2} P_J
                ld_f8(BB + r * 128 + c0, acc);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] *= kp[i];
                if (I < 3) st16(sm + S_B + btile_off(I + 1), tc::sw128_kmajor(r, c0, 16 * (I + 2)), acc);
                if (I < 2) {
                    ld_f8(gOff2 + I * 128 + c0, t8);
#pragma unroll
                    for (int i = 0; i < 8; ++i) t8[i] *= acc[i];
                    st16(sm + S_B + btile_off(I + 2), tc::sw128_kmajor(r, c0, 16 * (I + 3)), t8);
                }
                if (I < 1) {
                    ld_f8(gOff3 + I * 128 + c0, t8);
#pragma unroll
                    for (int i = 0; i < 8; ++i) t8[i] *= acc[i];
                    st16(sm + S_B + btile_off(3), tc::sw128_kmajor(r, c0, 64), t8);
                }
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            __syncthreads();
            tc::tc_fence_after();

            // ======== B: A and M block-rows on the tensor cores (overlaps A3b) ========
            if (tid == 0) {
                const uint32_t l0 = tc::smem_u32(sm + S_L), b0 = tc::smem_u32(sm + S_B);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
                    for (int J = 0; J < 4; ++J) {
                        const int n = 16 * (J + 1);
                        const uint64_t ad = tc::smem_desc_sw128(l0 + 4096 * J + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                        const uint64_t bd = tc::smem_desc_sw128(b0 + btile_off(J) + (ks >> 2) * n * 128 + (ks & 3) * 32, 16, 1024);
                        tc::mma_bf16(tmem + amcol(J), ad, bd, tc::idesc_bf16_f32(64, n, 0, 0), ks > 0 ? 1u : 0u);
                    }
                }
                tc::mma_commit(bar);
            }

            // A3b: K_end = k' bb KEF, K_gamma = |gamma_r| k', Q_gamma = |gamma_r| q'
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int c0 = hh ? cB : cA;
                const float* qx = hh ? qb : qa;
                const float* kx = hh ? kb : ka;
                float fb[8], kp[8], qp[8], acc[8], t8[8];
                ld_f8(FB + r * 128 + c0, fb);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float sg = signbit(fb[i]) ? -1.f : 1.f;
                    kp[i] = kx[i] * fk * sg;
                    qp[i] = qx[i] * fq * sg;
                    fb[i] = fabsf(fb[i]);
                }
                ld_f8(BB + r * 128 + c0, acc);
                ld_f8(gKef + I * 128 + c0, t8);
#pragma unroll
                for (int i = 0; i < 8; ++i) t8[i] *= acc[i] * kp[i];
                st16(sm + S_KE, tc::sw128_mnmajor(r, c0, 64), t8);
                ld_f8(gPre + I * 128 + c0, acc);
#pragma unroll
                for (int i = 0; i < 8; ++i) { acc[i] *= fb[i]; t8[i] = acc[i] * kp[i]; }
                st16(sm + S_KG, tc::sw128_mnmajor(r, c0, 64), t8);
#pragma unroll
                for (int i = 0; i < 8; ++i) t8[i] = acc[i] * qp[i];
                st16(sm + S_QG, tc::sw128_kmajor(r, c0, 64), t8);
            }
        }
        tc::mbar_wait(bar, phase & 1, abort_flag);
        ++phase;
        tc::tc_fence_after();
        {
            // M = 64 accumulator of block-row J: k rows in lanes 0..15, q rows in lanes 32..47.
            // Warp w reads TMEM lanes 32 (w % 4) ..: w % 4 == 0 -> A part, 1 -> M part; J = w / 4.
            const int quarter = warp & 3, J = warp >> 2;
            if (quarter < 2) {
                const int n = 16 * (J + 1);
                const int r = 16 * J + (lane & 15);
                for (int c0 = 0; c0 < n; c0 += 16) {
                    float x[16];
                    tc::tmem_ld16_sync(tc::tmem_addr(tmem, 32 * quarter, amcol(J) + c0), x);
                    if (lane < 16) {
                        if (quarter == 0) {
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
                }
                if (lane < 16) {
                    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    for (int j = n; j < 64; j += 8) {
                        if (quarter == 0) {
                            *reinterpret_cast<float4*>(sA + r * kStrideA + j) = make_float4(0.f, 0.f, 0.f, 0.f);
                            *reinterpret_cast<float4*>(sA + r * kStrideA + j + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
                        } else {
                            st16(sM, tc::sw128_kmajor(r, j, 64), z);
                        }
                    }
                }
            }
        }
        tc::tc_fence_before();
        __syncthreads();

        // exact recomputation of diagonal blocks whose gate total fell below 2^-60 (rare)
        for (int J = 0; J < 4; ++J) {
            if (!unsafe[J]) continue;
            float* fq = reinterpret_cast<float*>(sm + S_FQ);
            float* fk = reinterpret_cast<float*>(sm + S_FK);
            {
                const int rl = warp, r = 16 * J + rl;
                if (r < nvalid)
                    fallback_row(q, k, alpha, row0, rs, r, lane, rp, pos_offset + t0 + r, l2norm,
                                 fq + rl * 128, fk + rl * 128);
                else
                    for (int c = lane; c < 128; c += 32) fq[rl * 128 + c] = fk[rl * 128 + c] = 0.f;
            }
            __syncthreads();
            for (int pr = tid; pr < 136; pr += 512) {
                int rl = 0;
                while ((rl + 1) * (rl + 2) / 2 <= pr) ++rl;
                const int jl = pr - rl * (rl + 1) / 2;
                const int r = 16 * J + rl, j = 16 * J + jl;
                float accA = 0.f, accM = 0.f;
                for (int c = 0; c < kDK; ++c) {
                    float f = 1.f;
                    for (int tau = j + 1; tau <= r; ++tau)
                        f *= tau < nvalid ? fabsf(alpha[(row0 + tau * rs) * kDK + c]) : 1.f;
                    const float kj = fk[jl * 128 + c] * f;
                    accA += fk[rl * 128 + c] * kj;
                    accM += fq[rl * 128 + c] * kj;
                }
                sA[r * kStrideA + j] = j < r ? sb[r] * accA : 0.f;
                *reinterpret_cast<__nv_bfloat16*>(sM + tc::sw128_kmajor(r, j, 64)) = __float2bfloat16_rn(accM);
            }
            __syncthreads();
        }

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
        {
            float* sPt = reinterpret_cast<float*>(sm + S_PT);
            t_offdiag_level<1>(sA, sT, sX, sPt, tid);
            t_offdiag_level<2>(sA, sT, sX, sPt, tid);
            t_offdiag_level<3>(sA, sT, sX, sPt, tid);
        }
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
        if (tid == 0) {
            const uint32_t a0 = tc::smem_u32(sm + S_TB);
            const uint32_t kg = tc::smem_u32(sm + S_KG), vv = tc::smem_u32(sm + S_V);
            const uint32_t idesc = tc::idesc_bf16_f32(64, 128, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = tc::smem_desc_sw128(a0 + ks * 32, 16, 1024);
                tc::mma_bf16(tmem, ad, tc::smem_desc_sw128(kg + ks * 2048, 8192, 1024), idesc, ks > 0);
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
        // ======== G: results into the shared staging image, then one bulk store ========
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
                            unpack8(*reinterpret_cast<const uint4*>(sm + S_QG + tc::sw128_kmajor(r, n, 64)), qg);
#pragma unroll
                            for (int i = 0; i < 8; ++i) qg[i] -= x[c0 + i];
                            st16(out, WS_QP + tc::sw128_kmajor(r, n, 64), qg);
                        } else {
                            st16(out, WS_TILES + (n >> 5) * WS_TILE + WS_TILE_O + (r * 32 + (n & 31)) * 2, x + c0);
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
                        st16(out, WS_AC + tc::sw128_kmajor(cr, n, 128), y);
                    } else {
                        st16(out, WS_TILES + (n >> 5) * WS_TILE + (cr * 32 + (n & 31)) * 2, x + c0);
                    }
                }
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
        if (tid == 0) {
            tc::bulk_s2g(wsc, out, WS_CHUNK);
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
