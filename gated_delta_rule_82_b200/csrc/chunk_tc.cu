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
// Factor role (ckda_tc_intra alone, or the factor CTAs of ckda_tc_fused) -- persistent, one CTA
// of 512 threads per SM, loops over chunk-heads in head groups, chunk-major inside a group:
//   A  global loads of the next chunk-head issued together (and the one after prefetched into
//      L2); channel pass (thread per channel and 16-row block) forms the signed prefix gamma_r;
//      row pass (thread per row and two 8-channel groups, a RoPE pair) rotates and normalises q, k,
//      absorbs the signs and writes L, R, K_end with 16-byte stores.
//   B  tcgen05: [A | M] = L R^T  (M = 128, N = 64, K = 128), read back by all 16 warps.
//   C  T = (I + A)^-1 by blocked forward substitution in fp32; T' = T diag(beta) in bf16.
//   D  tcgen05: W^T = K_gamma^T T'^T, U~^T = V^T T'^T (M = 128, N = 64).
//   F  tcgen05: M W (M = 64) and K_end^T W (M = 128).
//   G  A_c and Q' staged in shared memory and written with bulk (TMA) stores, next to K_end, U~^T
//      and M straight from their operand tiles; once they have landed the chunk-head's ready flag
//      goes up.
// State role (ckda_tc_state alone, or the chain CTAs of ckda_tc_fused) -- one CTA per head at a
// time (all 128 dv columns), serial over its chunks, with the state transposed in Tensor Memory:
// per chunk the accumulation D_c^T = U~^T K_end + S^T A_c^T (M = 128, N = 128), whose state-free
// first part is issued ahead and whose second part (K = 128) is on the critical path; its
// read-back is the next state (fp32, rounded to bf16 as the next operand).  One off-path
// accumulation D_o^T = S^T Q'^T + U~^T M^T becomes the chunk's output.
// The fused launch is cooperative (every CTA resident at once): a few chain CTAs follow the
// ready flags of their heads while the factor CTAs produce them, so the serial pass hides behind
// the chunk-parallel work instead of following it.
#include <cuda.h>
#include <mutex>
#include <cudaTypedefs.h>

#include "fastdiv.h"
#include "lanes.h"
#include "internal.cuh"
#include "tc_sm100.cuh"

namespace ckda {

namespace {

constexpr int kC = 64, kDK = 128, kDV = 128;

// ---- workspace image of one chunk-head (bytes) ------------------------------------------------
constexpr uint32_t WS_AC = 0;          // A_c bf16, K-major swizzled, 128 rows x 128
constexpr uint32_t WS_KE = 32768;      // K_end bf16, MN-major swizzled, 64 token rows x 128
constexpr uint32_t WS_UT = 49152;      // U~^T bf16, K-major swizzled, 128 dv rows x 64 tokens
constexpr uint32_t WS_QP = 65536;      // Q'  bf16, K-major swizzled, 64 rows x 128
constexpr uint32_t WS_M = 81920;       // M bf16, K-major swizzled, 64 x 64
constexpr uint32_t WS_CHUNK = 90112;
// The state pass loads [WS_AC, WS_QP) (A_c, K_end, U~^T) for its chain products and
// [WS_UT, WS_CHUNK) (U~^T, Q', M) for the output: U~^T goes into both stages.
constexpr uint32_t WS_CHAIN_BYTES = WS_QP - WS_AC, WS_OUT_BYTES = WS_CHUNK - WS_UT;
// Ready flags: one 32-bit word per chunk-head after the images, set to 1 once the chunk-head's
// images are complete in global memory (cleared before every forward).
__host__ __device__ constexpr size_t flags_offset(size_t n_chunk_heads) { return n_chunk_heads * WS_CHUNK; }

// ---- kernel 1 shared memory (bytes from a 1024-aligned base) ---------------------------------
constexpr uint32_t S_G = 0;          // alpha (TMA), then the signed prefix gamma (fp32 [64][128])
constexpr uint32_t S_QR = 32768;     // raw q (TMA), bf16 [64][128] row-major
constexpr uint32_t S_KR = 49152;     // raw k (TMA), bf16 [64][128] row-major
constexpr uint32_t S_L = 65536;      // L: rows 0..63 g k', rows 64..127 g q' (K-major, 128 rows)
constexpr uint32_t S_R = 98304;      // R = k' / g (K-major, 64 rows); later T', X, Y; then Q' image
constexpr uint32_t S_V = 114688;     // V (TMA, 128-byte swizzle = MN-major, 64 K-rows x 128)
constexpr uint32_t S_KE = 131072;    // K_end (MN-major, 64 x 128): the MN-major A of K_end^T
constexpr uint32_t S_M = 147456;     // M bf16 K-major 64 x 64
constexpr uint32_t S_A = 155648;     // A fp32 [64][68]
constexpr uint32_t S_T = 173056;     // T fp32 [64][68]
constexpr uint32_t S_W = 190464;     // W^T K-major 128 x 64  (exact path: log2 prefix fp32 [64][128]
constexpr uint32_t S_U = 206848;     // U~^T K-major 128 x 64  spanning S_W and S_U)
constexpr uint32_t S_SM = 223232;    // small arrays (below)
constexpr uint32_t S_BYTES = S_SM + 3584 + 1024;
constexpr int kStrideA = 68;         // fp32 row stride of A and T
// T solve scratch inside R (dead after the [A | M] product)
constexpr uint32_t S_TB = S_R;               // T' bf16 K-major 64 x 64
constexpr uint32_t S_X = S_R + 8192;         // X0, X1 fp32 [16][24] each
constexpr uint32_t S_Y = S_R + 11264;        // Y fp32 [32][40]
// staging of the chunk's workspace image, over buffers that are dead by then
// (K_end, U~^T and M are stored straight from S_KE, S_U and S_M)
constexpr uint32_t S_OUT_QP = S_R;            // Q' image (16 KB)
constexpr uint32_t S_OUT_AC = S_A;            // A_c image (32 KB, over A and part of T)
static_assert(S_OUT_AC + 32768 <= S_W, "the A_c image must stay clear of W and U~^T");
// small arrays
constexpr uint32_t SM_P = S_SM;                  // signed block totals of alpha, fp32 [4][128]
constexpr uint32_t SM_GC = S_SM + 2048;          // gamma_C fp32 [128] (signed)
constexpr uint32_t SM_B = S_SM + 2560;           // beta fp32 [64]
constexpr uint32_t SM_FLAGS = S_SM + 2816;       // exact flag, abort flag, TMEM slot, 5 mbarriers
constexpr uint32_t SM_FREQ = S_SM + 3072;        // RoPE frequencies, turns per position [64]
constexpr uint32_t kInBytes = 32768 + 2 * 16384; // alpha, q, k of one chunk-head
constexpr uint32_t kVBytes = 16384;

constexpr float kSafeDecay = 3.009265538105056e-36f;  // 2^-118
// The factor role's bulk stores (and their waits, and the ready flags) all go through one thread:
// bulk-store groups belong to the thread that commits them.  It sits in warp 15, which has no
// product to issue.
constexpr int kStoreTid = 480;

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
__device__ __forceinline__ void st_bf16(uint8_t* base, uint32_t off, float x) {
    *reinterpret_cast<__nv_bfloat16*>(base + off) = __float2bfloat16_rn(x);
}

// 1/x by the hardware approximation (about 1 ulp); the result is rounded to bf16 afterwards.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// v[lane] for a register array of 32 values, by a select tree on the lane bits (no local memory).
__device__ __forceinline__ float select_lane(const float* v, int lane) {
    float a[16], b[8], c[4], d[2];
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = (lane & 1) ? v[2 * i + 1] : v[2 * i];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = (lane & 2) ? a[2 * i + 1] : a[2 * i];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = (lane & 4) ? b[2 * i + 1] : b[2 * i];
#pragma unroll
    for (int i = 0; i < 2; ++i) d[i] = (lane & 8) ? c[2 * i + 1] : c[2 * i];
    return (lane & 16) ? d[1] : d[0];
}

// Device status word of the forward kernels: 0, or the first failure recorded since the host last
// read it (kStatus* below).  Read and cleared by ckda_last_device_status.
__device__ int g_tc_error;
// Upper bound (ns) of one wait of the state role (a ready flag, or an mbarrier that may
// legitimately wait for a whole head group to be produced); settable from the host.
constexpr unsigned long long kDefaultWaitNs = 4000000000ull;   // 4 s
__device__ unsigned long long g_wait_limit_ns = kDefaultWaitNs;
// Codes of the status word (the first failure since the last read is kept).
constexpr int kStatusFactorWait = 1;     // a wait of the factor role ran out
constexpr int kStatusStateWait = 2;      // a wait of the state role ran out
constexpr int kStatusPackedOffsets = 3;  // device cu_seqlens disagree with the host copy
__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_tc_error, 0, code); }

// Tensor maps of one forward call: q, k, v (bf16), alpha (fp32, or bf16 logits) and out (bf16)
// as 4-D arrays {channel, head, token, batch}; boxes of 64 tokens of one (batch, head).
struct TcMaps {
    CUtensorMap q, k, v, alpha, out;
};

// Issue the TMA loads of the chunk of batch b, value head h (q/k head hk) starting at token t0:
// alpha -> G, q -> QR, k -> KR on bar_in; V (two 64-column halves, 128-byte swizzle) on bar_v.
// Rows past the sequence end read as zeros.  alpha, the largest input, is read once (one value
// head), so its lines go first when L2 evicts (the workspace images stay).
__device__ __forceinline__ void issue_inputs(const TcMaps& m, uint8_t* sm, uint64_t* bar_in,
                                             int b, int h, int hk, int t0, int gate_logits) {
    // gate values: fp32 [64][128] into G; logits: bf16 [64][128] into the upper half of G
    tc::mbar_arrive_expect_tx(bar_in, gate_logits ? kInBytes - 16384 : kInBytes);
    tc::tma_load_4d_hint(sm + S_G + (gate_logits ? 16384 : 0), &m.alpha, 0, h, t0, b, bar_in,
                         tc::policy_evict_first());
    tc::tma_load_4d(sm + S_QR, &m.q, 0, hk, t0, b, bar_in);
    tc::tma_load_4d(sm + S_KR, &m.k, 0, hk, t0, b, bar_in);
}
__device__ __forceinline__ void issue_v(const TcMaps& m, uint8_t* sm, uint64_t* bar_v, int b,
                                        int h, int t0) {
    tc::mbar_arrive_expect_tx(bar_v, kVBytes);
    tc::tma_load_4d(sm + S_V, &m.v, 0, h, t0, b, bar_v);
    tc::tma_load_4d(sm + S_V + 8192, &m.v, 64, h, t0, b, bar_v);
}

// ---- T = (I + A)^-1 ----------------------------------------------------------------------------
// Merge products of 16 x 16 and 32 x 32 blocks run on the warp-level tensor-core instruction
// (mma.sync m16n8k8, tf32 operands rounded to nearest, fp32 accumulation): these blocks are below
// the smallest tcgen05 tile (M = 64).  tf32 keeps 10 mantissa bits (the results become bf16 T').
// The rounding (to nearest, ties away from zero) is integer arithmetic on the bit pattern: half a
// tf32 unit added to the magnitude, then the 13 dropped bits cleared (a carry into the exponent
// rounds up to the next binade) -- the operands are finite.
// Fragment layout (PTX ISA, mma.m16n8k8 .tf32), g = lane / 4, t = lane % 4:
//   A (16 x 8, row-major)  a0 = A[g][t], a1 = A[g+8][t], a2 = A[g][t+4], a3 = A[g+8][t+4]
//   B (8 x 8)              b0 = B[t][g], b1 = B[t+4][g]
//   C, D (16 x 8, fp32)    c0 = D[g][2t], c1 = D[g][2t+1], c2 = D[g+8][2t], c3 = D[g+8][2t+1]
__device__ __forceinline__ uint32_t to_tf32(float x) {
    return (__float_as_uint(x) + 0x1000u) & 0xffffe000u;
}
// c (+)= A[16 x K] B[K x 8]: A rows `lda` floats apart, B rows `ldb` floats apart (shared memory)
template <int K>
__device__ __forceinline__ void mma_tile_tf32(float c[4], const float* a, int lda, const float* b,
                                              int ldb, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        const uint32_t a0 = to_tf32(a[g * lda + k0 + t]), a1 = to_tf32(a[(g + 8) * lda + k0 + t]);
        const uint32_t a2 = to_tf32(a[g * lda + k0 + t + 4]), a3 = to_tf32(a[(g + 8) * lda + k0 + t + 4]);
        const uint32_t b0 = to_tf32(b[(k0 + t) * ldb + g]), b1 = to_tf32(b[(k0 + t + 4) * ldb + g]);
        asm volatile(
            "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
            "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}
// store a D fragment (times `s`) to fp32 rows `ld` apart
__device__ __forceinline__ void st_tile_f32(float* d, int ld, const float c[4], float s, int lane) {
    const int g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2*>(d + g * ld + 2 * t) = make_float2(s * c[0], s * c[1]);
    *reinterpret_cast<float2*>(d + (g + 8) * ld + 2 * t) = make_float2(s * c[2], s * c[3]);
}
// store -D diag(beta) as bf16 T' (K-major, 64 x 64) at rows r0.., columns n0..
__device__ __forceinline__ void st_tile_tb(uint8_t* sTB, int r0, int n0, const float c[4],
                                           const float* sb, int lane) {
    const int g = lane >> 2, t = lane & 3, n = n0 + 2 * t;
    const float b0 = sb[n], b1 = sb[n + 1];
    *reinterpret_cast<uint32_t*>(sTB + tc::sw128_kmajor(r0 + g, n, 64)) = pack_bf16(-c[0] * b0, -c[1] * b1);
    *reinterpret_cast<uint32_t*>(sTB + tc::sw128_kmajor(r0 + g + 8, n, 64)) = pack_bf16(-c[2] * b0, -c[3] * b1);
}

// T = (I + A)^-1 for the strictly lower-triangular 64 x 64 A (fp32), by block doubling over
// 16 x 16 blocks T_IJ (I, J = 0..3):
//   phase 0  diagonal blocks T_JJ by forward substitution (fp32, CUDA cores);
//   phase 1  X0 = A_10 T_00,  X1 = A_32 T_22,  Y = [A_{[2:4],0} T_00 | A_{[2:4],1} T_11];
//   phase 2  T_10 = -T_11 X0,  T_32 = -T_33 X1,  Y_left -= Y_right X0
//            (then Y = A_{[2:4],[0:2]} T_{[0:2],[0:2]}, since T_10 = -T_11 X0);
//   phase 3  T_{[2:4],[0:2]} = -T_{[2:4],[2:4]} Y.
// Each finished block is also written as T' = T diag(beta) in bf16 (K-major, 64 x 64), the A
// operand of the W and U~ products.  Phases 1-3 are 12, 8 and 8 warp tiles of 16 x 8 outputs.
// Strides keep the fragment loads free of bank conflicts: A and T rows 68 floats apart (A-side),
// X0, X1 rows 24 apart and Y rows 40 apart (B-side).
constexpr int kStrideX = 24, kStrideY = 40;
__device__ __forceinline__ void t_solve(const float* sA, float* sT, const float* sb, uint8_t* sTB,
                                        float* sX, float* sY, int tid) {
    float* sX0 = sX;                    // [16][24]
    float* sX1 = sX + 16 * kStrideX;    // [16][24]
    const int warp = tid >> 5, lane = tid & 31;
    // ---- phase 0: diagonal blocks (threads 0..63: block J = tid / 16, column l = tid % 16);
    // the others zero block (2,3) of T and the blocks of T' above the diagonal
    if (tid < 64) {
        const int J = tid >> 4, l = tid & 15, base = 16 * J;
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
        const float bl = sb[base + l];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            sT[(base + i) * kStrideA + base + l] = tcol[i];
            st_bf16(sTB, tc::sw128_kmajor(base + i, base + l, 64), tcol[i] * bl);
        }
    } else {
        const int e = tid - 64;   // 0..447
        if (e < 64) {             // T block (2,3): rows 32..47, columns 48..63
            const int rr = e >> 2, c4 = 4 * (e & 3);
            *reinterpret_cast<float4*>(sT + (32 + rr) * kStrideA + 48 + c4) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // T' above the diagonal blocks: 192 chunks of 8 columns
        // (rows 0..15: 6 chunks each, rows 16..31: 4, rows 32..47: 2)
        for (int u = e; u < 192; u += 448) {
            int r, c8;
            if (u < 96) { r = u / 6; c8 = 16 + 8 * (u % 6); }
            else if (u < 160) { r = 16 + (u - 96) / 4; c8 = 32 + 8 * ((u - 96) % 4); }
            else { r = 32 + (u - 160) / 2; c8 = 48 + 8 * ((u - 160) % 2); }
            *reinterpret_cast<uint4*>(sTB + tc::sw128_kmajor(r, c8, 64)) = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    // ---- phase 1: 12 tiles (warps 0..11)
    if (warp < 12) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        const int n = 8 * (warp & 1);
        if (warp < 6) {           // [X0; Y_left] = A_{[1:4],0} T_00: row tiles 16, 32, 48
            const int m = 16 + 16 * (warp >> 1);
            mma_tile_tf32<16>(c, sA + m * kStrideA, kStrideA, sT + n, kStrideA, lane);
            if (m == 16) st_tile_f32(sX0 + n, kStrideX, c, 1.f, lane);
            else st_tile_f32(sY + (m - 32) * kStrideY + n, kStrideY, c, 1.f, lane);
        } else if (warp < 10) {   // Y_right = A_{[2:4],1} T_11: row tiles 32, 48
            const int m = 32 + 16 * ((warp - 6) >> 1);
            mma_tile_tf32<16>(c, sA + m * kStrideA + 16, kStrideA, sT + 16 * kStrideA + 16 + n, kStrideA, lane);
            st_tile_f32(sY + (m - 32) * kStrideY + 16 + n, kStrideY, c, 1.f, lane);
        } else {                  // X1 = A_32 T_22
            mma_tile_tf32<16>(c, sA + 48 * kStrideA + 32, kStrideA, sT + 32 * kStrideA + 32 + n, kStrideA, lane);
            st_tile_f32(sX1 + n, kStrideX, c, 1.f, lane);
        }
    }
    __syncthreads();
    // ---- phase 2: 8 tiles (warps 0..7)
    if (warp < 8) {
        const int n = 8 * (warp & 1);
        if (warp < 2) {           // T_10 = -T_11 X0 (T' only)
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            mma_tile_tf32<16>(c, sT + 16 * kStrideA + 16, kStrideA, sX0 + n, kStrideX, lane);
            st_tile_tb(sTB, 16, n, c, sb, lane);
        } else if (warp < 4) {    // T_32 = -T_33 X1 (T and T')
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            mma_tile_tf32<16>(c, sT + 48 * kStrideA + 48, kStrideA, sX1 + n, kStrideX, lane);
            st_tile_f32(sT + 48 * kStrideA + 32 + n, kStrideA, c, -1.f, lane);
            st_tile_tb(sTB, 48, 32 + n, c, sb, lane);
        } else {                  // Y_left -= Y_right X0: row tiles 0, 16 of Y
            const int m = 16 * ((warp - 4) >> 1);
            const int g = lane >> 2, t = lane & 3;
            float* y = sY + m * kStrideY + n;
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            mma_tile_tf32<16>(c, sY + m * kStrideY + 16, kStrideY, sX0 + n, kStrideX, lane);
            const float2 y0 = *reinterpret_cast<const float2*>(y + g * kStrideY + 2 * t);
            const float2 y1 = *reinterpret_cast<const float2*>(y + (g + 8) * kStrideY + 2 * t);
            const float d[4] = {y0.x - c[0], y0.y - c[1], y1.x - c[2], y1.y - c[3]};
            st_tile_f32(y, kStrideY, d, 1.f, lane);
        }
    }
    __syncthreads();
    // ---- phase 3: T_{[2:4],[0:2]} = -T_{[2:4],[2:4]} Y, 8 tiles (warps 0..7), T' only
    if (warp < 8) {
        const int m = 16 * (warp >> 2), n = 8 * (warp & 3);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        mma_tile_tf32<32>(c, sT + (32 + m) * kStrideA + 32, kStrideA, sY + n, kStrideY, lane);
        st_tile_tb(sTB, 32 + m, n, c, sb, lane);
    }
}

// Order in which the factor role visits the chunk-heads: heads in groups of G, and inside a
// group chunk by chunk (chunk c of every head of the group before chunk c + 1), so that the serial
// chains of a group, which consume their chunks in order, can run behind the factor work.  Item i
// is chunk c of batch*head bh (workspace chunk-head bh * NT + c).  The divisions go through
// multiply-shift forms of the launch's fixed divisors.
struct Item {
    int bh, c, b, h, hk;   // hk: the q/k head of value head h
};
struct WorkOrder {
    int G, last_g;
    FastDiv per;     // G * NT items per group
    FastDiv gfull;   // G heads in a group
    FastDiv glast;   // heads in the last group
    FastDiv heads;   // H
    FastDiv group;   // value heads per q/k head
    __device__ __forceinline__ Item item(int i) const {
        const uint32_t g = fastdiv(per, (uint32_t)i);
        const uint32_t r = (uint32_t)i - g * per.d;
        const FastDiv& gs = (int)g == last_g ? glast : gfull;
        const uint32_t c = fastdiv(gs, r);
        Item it;
        it.bh = (int)(g * (uint32_t)G + (r - c * gs.d));
        it.c = (int)c;
        it.b = (int)fastdiv(heads, (uint32_t)it.bh);
        it.h = it.bh - it.b * (int)heads.d;
        it.hk = (int)fastdiv(group, (uint32_t)it.h);
        return it;
    }
    // packed sequences: item i is entry i of the item table, (head unit, chunk of its lane)
    __device__ __forceinline__ Item item(int i, const int2* __restrict__ itab) const {
        if (!itab) return item(i);
        const int2 e = itab[i];
        Item it;
        it.bh = e.x;
        it.c = e.y;
        it.b = (int)fastdiv(heads, (uint32_t)it.bh);   // the lane
        it.h = it.bh - it.b * (int)heads.d;
        it.hk = (int)fastdiv(group, (uint32_t)it.h);
        return it;
    }
};
// The items one factor CTA takes: a leading run start1, start1 + stride1, ... (n1 of them), then
// start2, start2 + stride2, ... up to `total` (none when start2 >= total).
struct ItemSeq {
    int start1, stride1, n1, start2, stride2, total;
    __device__ __forceinline__ int at(int k) const {
        const int i = k < n1 ? start1 + k * stride1 : start2 + (k - n1) * stride2;
        return i < total ? i : -1;
    }
};
// Packed sequences of different lengths.  The sequences are dealt, in order, to lanes: runs of
// whole sequences with about the same number of chunks.  A lane plays the part of a batch row:
// head unit bh = lane * H + h, and chunk c of a unit is chunk c of its lane (the chunks of the
// lane's sequences in turn).  Lanes hold different numbers of chunks (lane_cnt); NT is the
// largest, and slots past a lane's count are never used.  Entry lane * NT + c of the chunk table
// (built on the device from the token offsets) says where a chunk lies: x = first token on the
// packed token axis, y = tokens in the chunk (1..64), z = its sequence, w = its index within the
// sequence, with kLastChunk set on the sequence's last chunk.  The item table lists the factor
// work, (unit, chunk) pairs, in the order the work order would give (head groups, chunk-major
// inside a group), skipping the unused slots.  Without tables (a batch of equal lengths) chunk c
// starts at token 64 c of batch row b.
constexpr int kLastChunk = 1 << 30;
struct PackedTabs {
    const int4* ctab;      // chunk table [lanes * NT]
    const int* lane_cnt;   // chunks of each lane [lanes]
    const int2* itab;      // item table [items]
};
struct ChunkAt {
    int b;            // batch coordinate of the tensor maps (0 for packed sequences)
    int t0, nvalid, seq, last;
    long long pos0;   // rotary position of the chunk's first token
};
__device__ __forceinline__ ChunkAt chunk_at(const int4* __restrict__ ctab, const Item& it, int T_len,
                                            int NT, long long pos_offset) {
    ChunkAt a;
    const int c = it.c;
    if (ctab) {
        const int4 e = ctab[(size_t)it.b * NT + c];   // it.b is the lane
        a.b = 0;
        a.t0 = e.x;
        a.nvalid = e.y;
        a.seq = e.z;
        a.last = (e.w & kLastChunk) != 0;
        a.pos0 = pos_offset + (long long)(e.w & (kLastChunk - 1)) * kC;
    } else {
        a.b = it.b;
        a.t0 = c * kC;
        a.nvalid = min(kC, T_len - a.t0);
        a.seq = 0;
        a.last = c == NT - 1;
        a.pos0 = pos_offset + a.t0;
    }
    return a;
}

inline WorkOrder make_work_order(int NT, int BH, int H, int G, int qk_group) {
    WorkOrder w;
    w.G = G;
    w.group = make_fastdiv((uint32_t)qk_group);
    w.last_g = (BH - 1) / G;
    w.per = make_fastdiv((uint32_t)(G * NT));
    w.gfull = make_fastdiv((uint32_t)G);
    w.glast = make_fastdiv((uint32_t)(BH - w.last_g * G));
    w.heads = make_fastdiv((uint32_t)H);
    return w;
}

// Ready flags.  The writer waits for its bulk stores to complete, orders them before the flag
// (proxy fence, then a release store at GPU scope); a reader acquires the flag and fences before
// its own bulk (async-proxy) loads of the images.
__device__ __forceinline__ void publish_ready(int* flag) {
    asm volatile("fence.proxy.async.global;" ::: "memory");
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(1u) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const int* flag) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    return v;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// Waits of the state role can last as long as the factor role takes to produce a head group
// (milliseconds on long sequences), so they are bounded by time (g_wait_limit_ns, read once per
// kernel into `limit`) rather than by a poll count.
__device__ __forceinline__ bool flag_wait(const int* flag, volatile int* abort, uint64_t limit) {
    if (ld_acquire(flag) != 0) {
        asm volatile("fence.proxy.async.global;" ::: "memory");
        return true;
    }
    const uint64_t t0 = global_ns();
    for (;;) {
        if (ld_acquire(flag) != 0) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            return true;
        }
        if (*abort) return false;
        if (global_ns() - t0 > limit) { *abort = 1; return false; }
        __nanosleep(256);
    }
}
__device__ __forceinline__ bool mbar_wait_long(uint64_t* bar, uint32_t parity, volatile int* abort,
                                               uint64_t limit) {
    if (tc::mbar_try_wait(bar, parity)) return true;   // the common case reads no timer
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0;; ++i) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if ((i & 255) == 255 && global_ns() - t0 > limit) { *abort = 1; return false; }
    }
}

// ---- the factor role: chunk-heads wo.item(i) for the items i of `seq` -----------------------------
// kLogits: alpha and beta hold logits (alpha = 2 sigma(a) - 1 from bf16 a, beta = 2 sigma(b)).
template <bool kLogits>
__device__ __forceinline__ void intra_role(uint8_t* sm, const TcMaps& maps, const void* __restrict__ alpha,
                                           const float* __restrict__ beta, uint8_t* __restrict__ ws,
                                           int* __restrict__ flags, PackedTabs pt,
                                           int T_len, int H, int NT, WorkOrder wo, ItemSeq seq, int l2norm,
                                           const RopeParams& rp, long long pos_offset, uint32_t tmem) {
    constexpr int gate_logits = kLogits ? 1 : 0;
    float* G = reinterpret_cast<float*>(sm + S_G);
    float* gP = reinterpret_cast<float*>(sm + SM_P);
    float* gGC = reinterpret_cast<float*>(sm + SM_GC);
    float* sb = reinterpret_cast<float*>(sm + SM_B);
    int* exact_path = reinterpret_cast<int*>(sm + SM_FLAGS);
    volatile int* abort_flag = exact_path + 4;
    uint64_t* bar = reinterpret_cast<uint64_t*>(exact_path + 16);   // tensor-core completions
    uint64_t* bar_in = bar + 1;                                     // alpha, q, k landed
    uint64_t* bar_v = bar + 2;                                      // V landed
    uint64_t* bar_w = bar + 3;                                      // W^T product complete
    uint64_t* bar_q = bar + 4;                                      // M W (for Q') complete
    float* sA = reinterpret_cast<float*>(sm + S_A);
    float* sT = reinterpret_cast<float*>(sm + S_T);
    float* sLg = reinterpret_cast<float*>(sm + S_W);   // exact path only
    uint8_t* sM = sm + S_M;
    uint8_t* sL = sm + S_L;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t rs = (size_t)H;   // stride between tokens, in rows of [B*T*H]
    tc::grid_launch_dependents();   // the state pass may start its set-up early

    // RoPE frequencies in shared memory: lanes index them by channel group, and a
    // per-lane index into the kernel-parameter array would serialise in the constant cache
    unsigned long long* sfreq = reinterpret_cast<unsigned long long*>(sm + SM_FREQ);
    if (tid < 64) sfreq[tid] = rp.turns[tid];
    if (tid == 32) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(bar_in, 1);
        tc::mbar_init(bar_v, 1);
        tc::mbar_init(bar_w, 1);
        tc::mbar_init(bar_q, 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    uint32_t phase = 0;   // completions of `bar` so far
    // the set-up above may overlap the previous kernel in the stream; from here on the kernel
    // reads the caller's inputs and writes the workspace, so it waits for that kernel
    tc::grid_dependency_wait();
    const int i0 = seq.at(0);
    if (tid == 0 && i0 >= 0) {
        tc::prefetch_tensormap(&maps.q);
        tc::prefetch_tensormap(&maps.k);
        tc::prefetch_tensormap(&maps.v);
        tc::prefetch_tensormap(&maps.alpha);
        const Item first = wo.item(i0, pt.itab);
        const ChunkAt fa = chunk_at(pt.ctab, first, T_len, NT, pos_offset);
        issue_inputs(maps, sm, bar_in, fa.b, first.h, first.hk, fa.t0, gate_logits);
        issue_v(maps, sm, bar_v, fa.b, first.h, fa.t0);
    }
    // the current item and where its chunk lies; the next item's entries are read one item
    // ahead, so that no table read sits at the top of an item
    Item item_next = wo.item(i0 >= 0 ? i0 : 0, pt.itab);
    ChunkAt at_next = chunk_at(pt.ctab, item_next, T_len, NT, pos_offset);

    // persistent loop over items; chunk-head ci = (batch*head) * NT + chunk
    uint32_t it = 0;
    int pending = -1;   // chunk-head whose images are stored but not yet flagged ready
    for (int k = 0, i = i0; i >= 0; i = seq.at(++k), ++it) {
        const Item cur = item_next;
        const int ci = cur.bh * NT + cur.c;
        const ChunkAt at = at_next;
        const int t0 = at.t0;
        const int nvalid = at.nvalid;
        const int inext = seq.at(k + 1);
        const bool has_next = inext >= 0;
        const Item nxt = wo.item(has_next ? inext : i, pt.itab);
        item_next = nxt;
        at_next = chunk_at(pt.ctab, nxt, T_len, NT, pos_offset);
        uint8_t* wsc = ws + (size_t)ci * WS_CHUNK;
        const size_t row0 = ((size_t)at.b * T_len + t0) * H + cur.h;
        float bval = (tid < 64 && tid < nvalid) ? beta[row0 + tid * rs] : 0.f;
        if (kLogits && tid < 64 && tid < nvalid) bval = gate_beta(bval);   // beta = 2 sigma(b)

        tc::mbar_wait(bar_in, it & 1, abort_flag);

        // ======== A2: channel pass -- thread (channel c, 16-row block I): signed prefix ========
        // gamma_r as a running product within the block; the sign carries the parity (a signed
        // zero keeps it on underflow).  Rows past the sequence end are identity gates.
        const int cc = tid & 127, cI = tid >> 7;
        if (tid == 0) *exact_path = 0;
        {
            float av[16];
            if constexpr (kLogits) {
                // logits a (bf16) in the upper half of G: all of them into registers first, since
                // the fp32 rows written below cover the same bytes; alpha = 2 sigma(a) - 1
                const __nv_bfloat16* la = reinterpret_cast<const __nv_bfloat16*>(sm + S_G + 16384);
#pragma unroll
                for (int rl = 0; rl < 16; ++rl) av[rl] = gate_alpha(__bfloat162float(la[(16 * cI + rl) * 128 + cc]));
                __syncthreads();
            } else {
#pragma unroll
                for (int rl = 0; rl < 16; ++rl) av[rl] = G[(16 * cI + rl) * 128 + cc];
            }
            float p = 1.f;
#pragma unroll
            for (int rl = 0; rl < 16; ++rl) {
                const int r = 16 * cI + rl;
                p *= r < nvalid ? av[rl] : 1.f;
                G[r * 128 + cc] = p;
            }
            gP[cI * 128 + cc] = p;
        }
        __syncthreads();
        if (tid < 128) {
            // block prefix factors (the product of the earlier blocks' totals), in place
            const float p0 = gP[tid], p1 = gP[128 + tid], p2 = gP[256 + tid], p3 = gP[384 + tid];
            const float pre2 = p0 * p1, pre3 = pre2 * p2, gc = pre3 * p3;
            gP[tid] = 1.f;
            gP[128 + tid] = p0;
            gP[256 + tid] = pre2;
            gP[384 + tid] = pre3;
            gGC[tid] = gc;
            if (!(fabsf(gc) >= kSafeDecay)) *exact_path = 1;
        }
        if (tid < 64) sb[tid] = bval;
        // the previous chunk-head's first store group (the Q' image over R, tiles 0-1 over
        // K_end and M) must have finished reading before the row pass rewrites R and K_end
        if (tid == kStoreTid) tc::bulk_wait_read<1>();
        __syncthreads();
        const bool exact = *exact_path != 0;

        // ======== A3: row pass -- thread (row r, 8-channel groups g and g + 8) ========
        {
            const int r = tid >> 3, g = tid & 7;
            const int cA = 8 * g, cB = 64 + 8 * g;
            float qa[8], qb[8], ka[8], kb[8];
            {
                const uint8_t* qrow = sm + S_QR + r * 256;
                const uint8_t* krow = sm + S_KR + r * 256;
                unpack8(*reinterpret_cast<const uint4*>(qrow + 16 * g), qa);
                unpack8(*reinterpret_cast<const uint4*>(qrow + 128 + 16 * g), qb);
                unpack8(*reinterpret_cast<const uint4*>(krow + 16 * g), ka);
                unpack8(*reinterpret_cast<const uint4*>(krow + 128 + 16 * g), kb);
            }
            // row norms (the rotation preserves them): reduce over the 8 threads of the row
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                sq += qa[i] * qa[i] + qb[i] * qb[i];
                sk += ka[i] * ka[i] + kb[i] * kb[i];
            }
            sq = group_sum<8>(sq);
            sk = group_sum<8>(sk);
            if (rp.enabled && rp.rot_dims != kDK) {
                // partial rotation of channels 0..63 only (64..127 carried through)
                const long long pos = at.pos0 + r;
                if (rp.convention == 0) {
                    // pairs (c, c + 32), frequency c % 32: channels 8g + i of this thread pair with
                    // those of the thread 4 lanes away in the same row (group g ^ 4)
                    const bool first = g < 4;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float sn, cs;
                        rope_sincos(pos, sfreq[8 * (g & 3) + i], &sn, &cs);
                        const float yq = __shfl_xor_sync(0xffffffffu, qa[i], 4);
                        const float yk = __shfl_xor_sync(0xffffffffu, ka[i], 4);
                        qa[i] = first ? qa[i] * cs - yq * sn : qa[i] * cs + yq * sn;
                        ka[i] = first ? ka[i] * cs - yk * sn : ka[i] * cs + yk * sn;
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < 4; ++m) {   // pairs (c, c + 1), frequency c / 2, c < 64
                        float sn, cs;
                        rope_sincos(pos, sfreq[4 * g + m], &sn, &cs);
                        float x0 = qa[2 * m], x1 = qa[2 * m + 1];
                        qa[2 * m] = x0 * cs - x1 * sn; qa[2 * m + 1] = x1 * cs + x0 * sn;
                        x0 = ka[2 * m]; x1 = ka[2 * m + 1];
                        ka[2 * m] = x0 * cs - x1 * sn; ka[2 * m + 1] = x1 * cs + x0 * sn;
                    }
                }
            } else if (rp.enabled) {
                const long long pos = at.pos0 + r;
                if (rp.convention == 0) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {   // pairs (cA + i, cB + i), frequency 8g + i
                        float sn, cs;
                        rope_sincos(pos, sfreq[8 * g + i], &sn, &cs);
                        float x0 = qa[i], x1 = qb[i];
                        qa[i] = x0 * cs - x1 * sn; qb[i] = x1 * cs + x0 * sn;
                        x0 = ka[i]; x1 = kb[i];
                        ka[i] = x0 * cs - x1 * sn; kb[i] = x1 * cs + x0 * sn;
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < 4; ++m) {   // pairs (c, c + 1) inside each 8-channel group
                        float sn, cs;
                        rope_sincos(pos, sfreq[4 * g + m], &sn, &cs);
                        float x0 = qa[2 * m], x1 = qa[2 * m + 1];
                        qa[2 * m] = x0 * cs - x1 * sn; qa[2 * m + 1] = x1 * cs + x0 * sn;
                        x0 = ka[2 * m]; x1 = ka[2 * m + 1];
                        ka[2 * m] = x0 * cs - x1 * sn; ka[2 * m + 1] = x1 * cs + x0 * sn;
                        rope_sincos(pos, sfreq[32 + 4 * g + m], &sn, &cs);
                        x0 = qb[2 * m]; x1 = qb[2 * m + 1];
                        qb[2 * m] = x0 * cs - x1 * sn; qb[2 * m + 1] = x1 * cs + x0 * sn;
                        x0 = kb[2 * m]; x1 = kb[2 * m + 1];
                        kb[2 * m] = x0 * cs - x1 * sn; kb[2 * m + 1] = x1 * cs + x0 * sn;
                    }
                }
            }
            const float fq = l2norm ? rsqrtf(sq + kL2Eps) : 1.f;
            const float fk = l2norm ? rsqrtf(sk + kL2Eps) : 1.f;
            const int rb = r >> 4;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int c0 = hh ? cB : cA;
                const float* qx = hh ? qb : qa;
                const float* kx = hh ? kb : ka;
                float gm[8], pre[8], kp[8], qp[8], t8[8];
                ld_f8(G + r * 128 + c0, gm);       // block-local gamma
                ld_f8(gP + rb * 128 + c0, pre);    // product of the earlier blocks' totals
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    gm[i] *= pre[i];                          // gamma_r, signed
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
                        t8[i] = kp[i] * rcp_approx(gm[i]);               // k' / g
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
        // the rest of the previous chunk-head's images (over A, T, W and U) must be read out
        // before the [A | M] read-back or the exact path rewrites them
        if (tid == kStoreTid) tc::bulk_wait_read<0>();
        __syncthreads();
        tc::tc_fence_after();
        // alpha, q, k of this chunk-head are consumed: bring in the next one's.  Issued by warp 15
        // (a TMA issue costs its thread several hundred cycles) while warp 0 issues the product.
        if (tid == 480 && has_next) issue_inputs(maps, sm, bar_in, at_next.b, nxt.h, nxt.hk, at_next.t0, gate_logits);
        if (!exact) {
            // ======== B: [A | M] = L R^T on the tensor cores (M = 128, N = 64, K = 128) ========
            if (warp == 0) {
                const uint64_t ad = tc::smem_desc_sw128(tc::smem_u32(sL), 16, 1024);
                const uint64_t bd = tc::smem_desc_sw128(tc::smem_u32(sm + S_R), 16, 1024);
                const uint32_t idesc = tc::idesc_bf16_f32(128, 64, 0, 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc::mma_bf16_warp(tmem, tc::desc_add(ad, (ks >> 2) * 16384 + (ks & 3) * 32),
                                      tc::desc_add(bd, (ks >> 2) * 8192 + (ks & 3) * 32), idesc, ks > 0);
                tc::mma_commit_warp(bar);
            }
        }
        if (!exact) {
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
                    float a = 1.f;
                    if (r < nvalid) {
                        const size_t ia = (row0 + r * rs) * kDK + tid;
                        if constexpr (kLogits)
                            a = gate_alpha(__bfloat162float(static_cast<const __nv_bfloat16*>(alpha)[ia]));
                        else
                            a = static_cast<const float*>(alpha)[ia];
                    }
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
                st_bf16(sM, tc::sw128_kmajor(r, j, 64), accM);
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
                st_bf16(sm + S_KE, tc::sw128_mnmajor(r, c, 64), sC * exp2f(sLg[63 * 128 + c] - sLg[r * 128 + c]) * kv);
                *kr = __float2bfloat16_rn(gr * kv);
                *qr = __float2bfloat16_rn(gr * qv);
            }
        }
        __syncthreads();

        // ======== C: T = (I + A)^-1 (fp32), T' = T diag(beta) (bf16) ========
        t_solve(sA, sT, sb, sm + S_TB, reinterpret_cast<float*>(sm + S_X),
                reinterpret_cast<float*>(sm + S_Y), tid);
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();

        // ======== D: W^T = K_gamma^T T'^T, U~^T = V^T T'^T  (M = 128, N = 64 each, K = 64) ========
        // The transposed products put a channel (or dv column) in every TMEM lane.  K_gamma^T is
        // rows 0..63 of L read as an MN-major A operand (64-channel blocks 16 KB apart), V^T the
        // TMA-swizzled V tile (blocks 8 KB apart); T'^T is T' itself as a K-major B operand.
        if (warp == 0) {
            tc::mbar_wait(bar_v, it & 1, abort_flag);
            __syncwarp();
            const uint64_t bd = tc::smem_desc_sw128(tc::smem_u32(sm + S_TB), 16, 1024);
            const uint64_t kd = tc::smem_desc_sw128(tc::smem_u32(sL), 16384, 1024);
            const uint64_t vd = tc::smem_desc_sw128(tc::smem_u32(sm + S_V), 8192, 1024);
            const uint32_t idesc = tc::idesc_bf16_f32(128, 64, 1, 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_bf16_warp(tmem, tc::desc_add(kd, ks * 2048), tc::desc_add(bd, ks * 32), idesc, ks > 0);
            tc::mma_commit_warp(bar_w);   // W^T: its read-back starts while U~^T computes
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_bf16_warp(tmem + 64, tc::desc_add(vd, ks * 2048), tc::desc_add(bd, ks * 32), idesc, ks > 0);
            tc::mma_commit_warp(bar);
        }
        if ((warp >> 2) < 2) tc::mbar_wait(bar_w, it & 1, abort_flag);
        else tc::mbar_wait(bar, phase & 1, abort_flag);
        ++phase;
        tc::tc_fence_after();
        {
            // warp w: lanes 32 (w % 4) .. (channel, or dv column, c); 32-column slice w / 4:
            // slices 0, 1 -> W^T tokens 0..63, slices 2, 3 -> U~^T tokens 0..63.  Both tiles are
            // K-major (rows c, K = token): the B operand of M W, K_end^T W and K_end^T U~, and the
            // A operand of U~^T M^T.
            const int quarter = warp & 3, slice = warp >> 2;
            const int c = 32 * quarter + lane;
            uint8_t* dst = sm + (slice < 2 ? S_W : S_U);
            const int j0 = 32 * (slice & 1);
            float x[32];
            tc::tmem_ld32_sync(tc::tmem_addr(tmem, 32 * quarter, 32 * slice), x);
#pragma unroll
            for (int i = 0; i < 32; i += 8) st16(dst, tc::sw128_kmajor(c, j0 + i, 128), x + i);
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();

        // ======== F: M W (M = 64) -> Q', K_end^T W (M = 128) -> A_c ========
        // (B_c = K_end^T U~ and the chunk's own output M U~ are left to the state pass, which
        // forms them in fp32 accumulators from the K_end, U~^T and M images)
        if (warp == 0) {
            const uint64_t md = tc::smem_desc_sw128(tc::smem_u32(sm + S_M), 16, 1024);
            const uint64_t ked = tc::smem_desc_sw128(tc::smem_u32(sm + S_KE), 8192, 1024);
            const uint64_t wd = tc::smem_desc_sw128(tc::smem_u32(sm + S_W), 16, 1024);
            const uint32_t id_q = tc::idesc_bf16_f32(64, 128, 0, 0);
            const uint32_t id_c = tc::idesc_bf16_f32(128, 128, 1, 0);
            // M W first: the Q' read-back overlaps K_end^T W
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)                                  // M W
                tc::mma_bf16_warp(tmem, tc::desc_add(md, ks * 32), tc::desc_add(wd, ks * 32), id_q, ks > 0);
            tc::mma_commit_warp(bar_q);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)                                  // K_end^T W
                tc::mma_bf16_warp(tmem + 192, tc::desc_add(ked, ks * 2048), tc::desc_add(wd, ks * 32), id_c, ks > 0);
            tc::mma_commit_warp(bar);
        }
        // The previous chunk-head's stores, issued at its end, have landed by now: flag it ready.
        // The release behind the flag takes a memory round trip, which the storing thread (in a
        // warp with nothing else to do until M W completes) spends while the products run.
        if (tid == kStoreTid && pending >= 0) {
            tc::bulk_wait_all();
            publish_ready(flags + pending);
        }
        pending = -1;
        // V of this chunk-head was consumed by the W/U~ products: bring in the next one's, from
        // warp 14 while warp 0 issues these products
        if (tid == 448 && has_next) issue_v(maps, sm, bar_v, at_next.b, nxt.h, at_next.t0);
        tc::mbar_wait(bar_q, it & 1, abort_flag);
        tc::tc_fence_after();
        // ======== G: results into shared staging images, then bulk stores in two groups ========
        {
            const int quarter = warp & 3, slice = warp >> 2;
            // (1) Q' = Q_gamma - M W (M = 64 layout): rows 16 quarter + lane, 32-column slice
            {
                const int r = 16 * quarter + (lane & 15);
                float x[32];
                tc::tmem_ld32_sync(tc::tmem_addr(tmem, 32 * quarter, 32 * slice), x);
                if (lane < 16) {
#pragma unroll
                    for (int c0 = 0; c0 < 32; c0 += 8) {
                        const int n = 32 * slice + c0;
                        float qg[8];
                        unpack8(*reinterpret_cast<const uint4*>(sL + tc::sw128_kmajor(64 + r, n, 128)), qg);
#pragma unroll
                        for (int i = 0; i < 8; ++i) qg[i] -= x[c0 + i];
                        st16(sm + S_OUT_QP, tc::sw128_kmajor(r, n, 64), qg);
                    }
                }
            }
            // (2) A_c = Diag(gamma_C) - K_end^T W (M = 128, lane = row c'): warp w reads columns
            // 32 (w / 4) .. + 31 of rows 32 (w % 4) + lane
            tc::mbar_wait(bar, phase & 1, abort_flag);
            ++phase;
            tc::tc_fence_after();
            {
                const int cr = 32 * quarter + lane;
                const int n0 = 32 * slice;
                float x[32];
                tc::tmem_ld32_sync(tc::tmem_addr(tmem, 32 * quarter, 192 + n0), x);
                // the diagonal element of row cr lies in this slice when slice == quarter, at x[lane]
                const float dx = slice == quarter ? select_lane(x, lane) : 0.f;
#pragma unroll
                for (int c0 = 0; c0 < 32; c0 += 8) {
                    float y[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[i] = -x[c0 + i];
                    st16(sm + S_OUT_AC, tc::sw128_kmajor(cr, n0 + c0, 128), y);
                }
                if (slice == quarter) st_bf16(sm + S_OUT_AC, tc::sw128_kmajor(cr, cr, 128), gGC[cr] - dx);
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
        if (tid == kStoreTid) {
            // group 1: the images over buffers the next row pass rewrites first (Q' over R, K_end
            // straight from its operand tile)
            tc::bulk_s2g(wsc + WS_QP, sm + S_OUT_QP, 16384);
            tc::bulk_s2g(wsc + WS_KE, sm + S_KE, 16384);
            tc::bulk_commit();
            // group 2: A_c, then U~^T and M straight from their operand tiles
            tc::bulk_s2g(wsc + WS_AC, sm + S_OUT_AC, 32768);
            tc::bulk_s2g(wsc + WS_UT, sm + S_U, 16384);
            tc::bulk_s2g(wsc + WS_M, sm + S_M, 8192);
            tc::bulk_commit();
        }
        pending = ci;
    }
    if (tid == kStoreTid) {
        tc::bulk_wait_all();
        if (pending >= 0) publish_ready(flags + pending);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) record_status(kStatusFactorWait);
    // the CTA may go on to another role over this shared memory, whose copies (async proxy) must
    // come after this role's plain writes
    tc::fence_proxy_async_smem();
    if (tid == 32) {
        tc::mbar_inval(bar);
        tc::mbar_inval(bar_in);
        tc::mbar_inval(bar_v);
        tc::mbar_inval(bar_w);
        tc::mbar_inval(bar_q);
    }
    __syncthreads();
}

// ---- the state role: the serial pass over the chunks of heads head0, head0 + hstride, ... ---------
// One CTA of 512 threads carries whole heads (all 128 dv columns), one head after the other; its
// items u = k NT + c run over (head k of the CTA, chunk c).  The state is kept transposed: S^T
// (dv x dk) lives in Tensor Memory as the A operand of both products,
//     D_c^T = U~^T K_end + S^T A_c^T  (M = 128 dv, N = 128)         -> S_next^T = D_c^T
//     D_o^T = S^T Q'^T + U~^T M^T      (M = 128 dv, N = 64 tokens)  -> O^T = scale D_o^T
// so B_c = K_end^T U~ and the chunk's own output M U~ are accumulated in fp32 and never rounded.
// The U~^T K_end part needs no state: it is issued as soon as the epilogue has read the previous
// accumulator, while the epilogue is still rounding and writing S^T.
// Warp roles:
//   warps 0-7    chain epilogue: warp w owns dv columns 32 (w % 4) .. + 31 (its TMEM lanes) and
//                state rows 64 (w / 4) .. + 63; reads S_next^T in fp32 and writes it back into
//                TMEM as the bf16 operand of the next products (hT in fp32 after a head's last
//                chunk)
//   warp 8       chain issue
//   warp 9       output issue
//   warp 10      chain loads: A_c, K_end and U~^T of each item (one 64 KB bulk copy, two stages)
//   warp 11      output loads: U~^T, Q' and M of each item (one 40 KB bulk copy, two stages)
//   warps 12-15  output epilogue: lane = dv column; the chunk's 64 x 128 output tile goes through
//                a shared-memory staging tile and leaves with one tensor (TMA) store
// Only the chain roles are on the serial path.  The output product of item u is issued once the
// chain product of item u has completed, so it runs while the chain epilogue works.  S^T
// alternates between two TMEM buffers: S_{u+1}^T goes into the buffer of S_{u-1}^T once the
// output product of item u - 1 has read it.  Every load of an item waits for the item's ready
// flag, every role issues from a converged warp (one elected lane) and every wait is bounded.
constexpr uint32_t SS_C = 0;             // chain stages: A_c (32 KB), K_end (16 KB), U~^T (16 KB)
constexpr uint32_t SS_CSTAGE = WS_CHAIN_BYTES;
constexpr uint32_t SS_O = 2 * SS_CSTAGE; // output stages: U~^T (16 KB), Q' (16 KB), M (8 KB)
constexpr uint32_t SS_OSTAGE = WS_OUT_BYTES;
constexpr uint32_t SS_STG = SS_O + 2 * SS_OSTAGE;   // output tile bf16 [64 tokens][128 dv]
constexpr uint32_t SS_BAR = SS_STG + 16384;
constexpr uint32_t SS_BYTES = SS_BAR + 256 + 1024;
constexpr uint32_t FUSED_BYTES = SS_BYTES > S_BYTES ? SS_BYTES : S_BYTES;
static_assert(SS_OSTAGE % 1024 == 0 && (WS_QP - WS_UT) % 1024 == 0 && (WS_M - WS_UT) % 1024 == 0 &&
                  (WS_KE - WS_AC) % 1024 == 0 && (WS_UT - WS_AC) % 1024 == 0,
              "operand tiles of a stage must stay 1024-byte aligned");
// TMEM columns: D_c^T 0..127, S^T buffers of 64 (bf16 pairs) from 128, D_o^T buffers of 64 from 256
constexpr uint32_t kColS = 128, kColO = 256;

// ---- segments of the state pass (the segment-parallel chunk-transition scan) -------------------
// The NT chunks of every head unit form P segments of L chunks (the last one may be shorter).  A
// summary pass gives, for every segment s < P - 1, its end state E_s when entered with h0 (s = 0)
// or with zero (s > 0), and for 0 < s < P - 1 its transition F_s, the product of its A_c (a chain
// entered with the identity and without the B_c terms).  A scan then forms the state entering
// every segment, S_1 = E_0 and S_{s+1} = F_s S_s + E_s, and a second pass runs every segment from
// its entering state with its outputs.  States and transitions are fp32 [dk][dv] (or [dk][dk])
// arrays of the workspace, indexed (unit * P + s).
struct SegArgs {
    int P, L;
    int summary;          // 1: the summary pass (no outputs); 0: the pass with outputs
    float* segE;          // end states E_s
    float* segF;          // transitions F_s
    const float* segS;    // entering states S_s (S_0 = h0)
};
struct SegUnit {
    int bh, s, c0, c1;
    int transition;       // 1: a transition chain (identity start, no B_c terms)
};
__host__ __device__ inline int seg_units(const SegArgs& a, int BH) {
    return a.summary ? BH * (a.P - 1) + BH * (a.P > 2 ? a.P - 2 : 0) : BH * a.P;
}
// summary units: the end-state chains (unit, s < P - 1), then the transition chains
// (unit, 0 < s < P - 1); pass units: (unit, s)
__device__ __forceinline__ SegUnit seg_unit(const SegArgs& a, int vu, int BH, int NT) {
    SegUnit u;
    u.transition = 0;
    if (a.summary) {
        const int ne = BH * (a.P - 1);
        if (vu < ne) {
            u.bh = vu / (a.P - 1);
            u.s = vu % (a.P - 1);
        } else {
            u.transition = 1;
            u.bh = (vu - ne) / (a.P - 2);
            u.s = 1 + (vu - ne) % (a.P - 2);
        }
    } else {
        u.bh = vu / a.P;
        u.s = vu % a.P;
    }
    u.c0 = u.s * a.L;
    u.c1 = min(NT, u.c0 + a.L);
    return u;
}
// The items (unit, chunk) of the units first, first + stride, ... in order.
struct SegIter {
    SegArgs a;
    int BH, NT, vu, stride, nunits, c;
    SegUnit cur;
    __device__ SegIter(const SegArgs& a_, int first, int stride_, int BH_, int NT_)
        : a(a_), BH(BH_), NT(NT_), vu(first), stride(stride_), nunits(seg_units(a_, BH_)), c(0) {
        cur = SegUnit{0, 0, 0, 0, 0};
        if (vu < nunits) {
            cur = seg_unit(a, vu, BH, NT);
            c = cur.c0;
        }
    }
    __device__ bool unit_end() const { return c + 1 == cur.c1; }
    __device__ void next() {
        if (++c == cur.c1) {
            vu += stride;
            if (vu < nunits) {
                cur = seg_unit(a, vu, BH, NT);
                c = cur.c0;
            }
        }
    }
};

// kSeg: the items are the chunks of segment units (SegArgs) head0, head0 + hstride, ... instead of
// whole head units; in the summary pass there are no outputs.
template <bool kSeg>
__device__ __forceinline__ void state_role(uint8_t* sm, const TcMaps& maps, const uint8_t* __restrict__ ws,
                                           const int* __restrict__ flags, PackedTabs pt,
                                           const float* __restrict__ h0,
                                           __nv_bfloat16* __restrict__ out, float* __restrict__ hT,
                                           int T_len, int H, int NT, int BH, float scale, int head0,
                                           int hstride, uint32_t tmem, SegArgs sa) {
    uint64_t* full_c = reinterpret_cast<uint64_t*>(sm + SS_BAR);   // [2] A_c, K_end, U~^T landed
    uint64_t* empty_c = full_c + 2;     // [2] chain stage read by the chain products (commit)
    uint64_t* full_o = empty_c + 2;     // [2] Q', U~^T, M landed
    uint64_t* empty_o = full_o + 2;     // [2] output stage read by the output product (commit)
    uint64_t* mma_c = empty_o + 2;      // D_c^T complete
    uint64_t* s_ready = mma_c + 1;      // [2] S^T buffer written (8 epilogue warps)
    uint64_t* dc_done = s_ready + 2;    // [2] D_c^T of the item using S^T buffer b complete
    uint64_t* mma_o = dc_done + 2;      // [4] D_o^T complete
    uint64_t* o_free = mma_o + 4;       // [4] D_o^T read back (4 output-epilogue warps)
    uint64_t* dc_free = o_free + 4;     // D_c^T read back (8 chain-epilogue warps)
    volatile int* abort_flag = reinterpret_cast<volatile int*>(dc_free + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // chunks of head unit bh: NT, or (packed sequences) the count of its lane
    const int4* __restrict__ ctab = pt.ctab;
    auto units_chunks = [&](int bh) { return pt.lane_cnt ? pt.lane_cnt[bh / H] : NT; };
    int U = 0;   // items of this CTA: the chunks of heads head0, head0 + hstride, ...
    if constexpr (kSeg) {
        const int nu = seg_units(sa, BH);
        for (int vu = head0; vu < nu; vu += hstride) {
            const SegUnit su = seg_unit(sa, vu, BH, NT);
            U += su.c1 - su.c0;
        }
    } else {
        for (int bh = head0; bh < BH; bh += hstride) U += units_chunks(bh);
    }
    const bool outputs = !kSeg || !sa.summary;

    if (tid == 32) {
        tc::mbar_init(dc_free, 8);
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&full_c[s], 1);
            tc::mbar_init(&empty_c[s], 1);
            tc::mbar_init(&full_o[s], 1);
            tc::mbar_init(&empty_o[s], 1);
            tc::mbar_init(&s_ready[s], 8);
            tc::mbar_init(&dc_done[s], 1);
        }
        tc::mbar_init(mma_c, 1);
        for (int s = 0; s < 4; ++s) {
            tc::mbar_init(&mma_o[s], 1);
            tc::mbar_init(&o_free[s], 4);
        }
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    // a launch after the factor kernel waits for it here (no effect otherwise)
    tc::grid_dependency_wait();
    tc::grid_launch_dependents();
    const uint64_t limit = g_wait_limit_ns;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait_long(bar, parity, abort_flag, limit));
    };
    // items advance as (head k, chunk c) counters, so no step divides by NT

    if (warp < 8) {
        // ---- chain epilogue: lane = dv column n, state rows cb .. cb + 63 ----
        const int q = warp & 3, hf = warp >> 2;
        const int n = 32 * q + lane, cb = 64 * hf;
        float S[64];   // S[j] = S(cb + j, n)
        // state row of head unit bh at chunk c: the batch row's (b, h), or, for packed sequences
        // (bh = h), (sequence of chunk c, h)
        auto load_h0 = [&](int srow) {
            if (h0) {
                const float* src = h0 + ((size_t)srow * kDK + cb) * kDV + n;
#pragma unroll
                for (int j = 0; j < 64; ++j) S[j] = src[(size_t)j * kDV];
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) S[j] = 0.f;
            }
        };
        // S^T as the TMEM A operand: lane n, column 32 hf + j holds rows cb + 2j, cb + 2j + 1
        auto put_s = [&](int u) {
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = pack_bf16(S[2 * j], S[2 * j + 1]);
            tc::tmem_st32(tc::tmem_addr(tmem + kColS + 64 * (u & 1) + 32 * hf, 32 * q, 0), v);
            tc::tmem_st_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&s_ready[u & 1]);
        };
        if constexpr (kSeg) {
            // the state entering a segment unit: S_s (pass with outputs); h0 or zero (end-state
            // chains); the identity (transition chains)
            auto load_init = [&](const SegUnit& su) {
                const float* src = nullptr;
                if (!sa.summary)
                    src = sa.segS + ((size_t)su.bh * sa.P + su.s) * kDK * kDV;
                else if (!su.transition && su.s == 0 && h0)
                    src = h0 + (size_t)su.bh * kDK * kDV;
                if (src) {
                    src += (size_t)cb * kDV + n;
#pragma unroll
                    for (int j = 0; j < 64; ++j) S[j] = src[(size_t)j * kDV];
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j) S[j] = (su.transition && cb + j == n) ? 1.f : 0.f;
                }
            };
            SegIter it(sa, head0, hstride, BH, NT);
            if (U > 0) {
                load_init(it.cur);
                put_s(0);
            }
            for (int u = 0; u < U; ++u) {
                const bool unit_end = it.unit_end();
                if (!wait(mma_c, u & 1)) break;
                tc::tc_fence_after();
                tc::tmem_ld64_sync(tc::tmem_addr(tmem, 32 * q, cb), S);
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(dc_free);
                if (unit_end && !*abort_flag) {
                    // the pass writes hT after a head's last chunk; the summary its E_s or F_s
                    float* dst = nullptr;
                    if (!sa.summary)
                        dst = (hT && it.c == NT - 1) ? hT + (size_t)it.cur.bh * kDK * kDV : nullptr;
                    else
                        dst = (it.cur.transition ? sa.segF : sa.segE) +
                              ((size_t)it.cur.bh * sa.P + it.cur.s) * kDK * kDV;
                    if (dst) {
                        dst += (size_t)cb * kDV + n;
#pragma unroll
                        for (int j = 0; j < 64; ++j) dst[(size_t)j * kDV] = S[j];
                    }
                }
                if (u + 1 < U) {
                    if (outputs && u >= 1 && !wait(&mma_o[(u - 1) & 3], ((u - 1) >> 2) & 1)) break;
                    it.next();
                    if (unit_end) load_init(it.cur);
                    put_s(u + 1);
                } else {
                    tc::tc_fence_before();
                }
            }
        } else {
        // packed sequences: unit bh is (lane bh / H, head bh % H); tab is its lane's chunk table
        // and srow gives the state row of (sequence, head)
        const int4* tab = ctab ? ctab + (size_t)(head0 / H) * NT : nullptr;
        auto srow = [&](int4 e, int bh) { return ctab ? e.z * H + bh % H : bh; };
        int nc = U > 0 ? units_chunks(head0) : 0;
        if (U > 0) {
            load_h0(srow(ctab ? tab[0] : make_int4(0, 0, 0, 0), head0));
            put_s(0);
        }
        for (int u = 0, c = 0, bh = head0; u < U; ++u) {
            // this chunk's entry and the next item's (read ahead of the wait)
            const bool same = c + 1 < nc;
            const int c2 = same ? c + 1 : 0, bh2 = same ? bh : bh + hstride;
            const int4* tab2 = ctab ? (same ? tab : ctab + (size_t)(bh2 / H) * NT) : nullptr;
            const int4 ecur = ctab ? tab[c] : make_int4(0, 0, 0, c == NT - 1 ? kLastChunk : 0);
            const int4 enext = ctab && u + 1 < U ? tab2[c2] : make_int4(0, 0, 0, c2);
            if (!wait(mma_c, u & 1)) break;
            tc::tc_fence_after();
            tc::tmem_ld64_sync(tc::tmem_addr(tmem, 32 * q, cb), S);
            // the accumulator is read: the next item's state-free part may go in
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(dc_free);
            const bool last = (ecur.w & kLastChunk) != 0;
            if (last && hT && !*abort_flag) {
                float* dst = hT + ((size_t)srow(ecur, bh) * kDK + cb) * kDV + n;
#pragma unroll
                for (int j = 0; j < 64; ++j) dst[(size_t)j * kDV] = S[j];
            }
            if (u + 1 < U) {
                // the buffer of S_{u+1}^T held S_{u-1}^T: the output product of item u - 1 must
                // be done with it
                if (u >= 1 && !wait(&mma_o[(u - 1) & 3], ((u - 1) >> 2) & 1)) break;
                // the next item starts a sequence: its initial state
                if ((enext.w & (kLastChunk - 1)) == 0) load_h0(srow(enext, bh2));
                put_s(u + 1);
            } else {
                tc::tc_fence_before();
            }
            if (++c == nc) {
                c = 0;
                bh += hstride;
                tab = tab2;
                if (u + 1 < U) nc = units_chunks(bh);
            }
        }
        }
    } else if (warp == 8) {
        // ---- chain issue: D_c^T = U~^T K_end (both from the stage: K-major A, MN-major B) and
        // then + S^T A_c^T (A = S^T from TMEM, B = the K-major A_c image read as K-major B) ----
        const uint32_t idc = tc::idesc_bf16_f32(128, 128, 0, 0);
        const uint32_t idb = tc::idesc_bf16_f32(128, 128, 0, 1);
        const uint64_t k_desc0 = tc::smem_desc_sw128(tc::smem_u32(sm + SS_C + (WS_KE - WS_AC)), 8192, 1024);
        const uint64_t u_desc0 = tc::smem_desc_sw128(tc::smem_u32(sm + SS_C + (WS_UT - WS_AC)), 16, 1024);
        const uint64_t c_desc0 = tc::smem_desc_sw128(tc::smem_u32(sm + SS_C), 16, 1024);
        SegIter it(sa, head0, hstride, BH, NT);   // (segment units only)
        for (int u = 0; u < U; ++u) {
            const int st = u & 1;
            if (!wait(&full_c[st], (u >> 1) & 1)) break;
            // the epilogue has read the previous accumulator
            if (u >= 1 && !wait(dc_free, (u - 1) & 1)) break;
            tc::tc_fence_after();
            // a transition chain has no B_c = K_end^T U~ term
            bool bterm = true;
            if constexpr (kSeg) bterm = !it.cur.transition;
            if (bterm) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16_warp(tmem, tc::desc_add(u_desc0, st * SS_CSTAGE + ks * 32),
                                      tc::desc_add(k_desc0, st * SS_CSTAGE + ks * 2048), idb, ks > 0 ? 1u : 0u);
            }
            if (!wait(&s_ready[st], (u >> 1) & 1)) break;
            tc::tc_fence_after();
            const uint64_t bd = tc::desc_add(c_desc0, st * SS_CSTAGE);
            const uint32_t a = tmem + kColS + 64 * st;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_bf16_tmem_a_warp(tmem, a + 8 * ks, tc::desc_add(bd, (ks >> 2) * 16384 + (ks & 3) * 32),
                                         idc, (bterm || ks > 0) ? 1u : 0u);
            tc::mma_commit_warp(mma_c);
            tc::mma_commit_warp(&dc_done[st]);
            tc::mma_commit_warp(&empty_c[st]);
            if constexpr (kSeg) it.next();
        }
    } else if (warp == 9) {
        // ---- output issue: S^T Q'^T (A in TMEM) + U~^T M^T (both from shared memory) ----
        const uint32_t ido = tc::idesc_bf16_f32(128, 64, 0, 0);
        const uint64_t o_desc0 = tc::smem_desc_sw128(tc::smem_u32(sm + SS_O), 16, 1024);
        for (int u = 0; u < (outputs ? U : 0); ++u) {
            const int st = u & 1, ob = u & 3;
            if (!wait(&full_o[st], (u >> 1) & 1)) break;
            // issued once D_c(u) has completed, so it never shares the tensor pipe with a chain
            // product; S_u^T is complete since D_c(u) read it
            if (!wait(&dc_done[st], (u >> 1) & 1)) break;
            if (u >= 4 && !wait(&o_free[ob], ((u >> 2) - 1) & 1)) break;
            tc::tc_fence_after();
            const uint64_t od = tc::desc_add(o_desc0, st * SS_OSTAGE);
            const uint32_t d = tmem + kColO + 64 * ob;
            const uint32_t a = tmem + kColS + 64 * st;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)                                  // S^T Q'^T
                tc::mma_bf16_tmem_a_warp(d, a + 8 * ks,
                                         tc::desc_add(od, (WS_QP - WS_UT) + (ks >> 2) * 8192 + (ks & 3) * 32),
                                         ido, ks > 0 ? 1u : 0u);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)                                  // + U~^T M^T
                tc::mma_bf16_warp(d, tc::desc_add(od, ks * 32), tc::desc_add(od, (WS_M - WS_UT) + ks * 32),
                                  ido, 1u);
            tc::mma_commit_warp(&mma_o[ob]);
            tc::mma_commit_warp(&empty_o[st]);
        }
    } else if (warp == 10 || warp == 11) {
        // ---- loads: warp 10 the chain stages, warp 11 the output stages ----
        if (lane == 0 && (warp == 10 || outputs)) {
            const bool chain = warp == 10;
            uint64_t* fullb = chain ? full_c : full_o;
            uint64_t* emptyb = chain ? empty_c : empty_o;
            const uint32_t bytes = chain ? SS_CSTAGE : SS_OSTAGE;
            uint8_t* stage0 = sm + (chain ? SS_C : SS_O);
            int issued = 0;
            int nc = U > 0 && !kSeg ? units_chunks(head0) : 0;
            SegIter it(sa, head0, hstride, BH, NT);   // (segment units only)
            for (int c = 0, bh = head0; issued < U; ++issued) {
                const int st = issued & 1;
                if (issued >= 2 && !mbar_wait_long(&emptyb[st], ((issued >> 1) - 1) & 1, abort_flag, limit))
                    break;
                size_t ci;
                if constexpr (kSeg) {
                    ci = (size_t)it.cur.bh * NT + it.c;
                    it.next();
                } else {
                    ci = (size_t)bh * NT + c;
                    if (++c == nc) {
                        c = 0;
                        bh += hstride;
                        if (issued + 1 < U) nc = units_chunks(bh);
                    }
                }
                if (!flag_wait(flags + ci, abort_flag, limit)) break;
                tc::mbar_arrive_expect_tx(&fullb[st], bytes);
                tc::bulk_g2s(stage0 + st * bytes, ws + ci * WS_CHUNK + (chain ? WS_AC : WS_UT), bytes,
                             &fullb[st]);
            }
            if (*abort_flag) {
                // let every copy still in flight land before the shared memory is released
                for (int c = issued > 2 ? issued - 2 : 0; c < issued; ++c)
                    for (uint32_t i = 0; i < tc::kSpinLimit; ++i)
                        if (tc::mbar_try_wait(&fullb[c & 1], (c >> 1) & 1)) break;
            }
        }
    } else {
        // ---- output epilogue: warp 12 + q reads TMEM lanes 32 q .. (dv columns n) ----
        // The four warps move in step (named barrier 1): they leave the loop together, on a
        // vote, so that none waits at a barrier the others have left.
        const int q = warp & 3, n = 32 * q + lane;
        const bool leader = warp == 12 && lane == 0;
        uint8_t* stg = sm + SS_STG;
        const int4* otab = ctab ? ctab + (size_t)(head0 / H) * NT : nullptr;   // the lane's table
        int nc = U > 0 && !kSeg ? units_chunks(head0) : 0;
        SegIter it(sa, head0, hstride, BH, NT);   // (segment units only)
        for (int u = 0, c = 0, bh = head0; u < (outputs ? U : 0); ++u) {
            const int ob = u & 3;
            if constexpr (kSeg) {
                c = it.c;
                bh = it.cur.bh;
            }
            // the chunk's first token and length (packed sequences: from the chunk table)
            const int4 e = ctab ? otab[c] : make_int4(c * kC, kC, 0, 0);
            const bool ok = mbar_wait_long(&mma_o[ob], (u >> 2) & 1, abort_flag, limit);
            // the previous item's tensor store must be done reading the staging tile
            if (leader) tc::bulk_wait_read<0>();
            __syncwarp();
            if (tc::bar_any(1, 128, !ok)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float d[32];
                tc::tmem_ld32_sync(tc::tmem_addr(tmem + kColO + 64 * ob, 32 * q, 32 * half), d);
                if (half == 1) {
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&o_free[ob]);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    st_bf16(stg, (32 * half + i) * 256 + 2 * n, scale * d[i]);
            }
            tc::fence_proxy_async_smem();
            __syncwarp();
            tc::bar_named(1, 128);
            const int h = bh % H;
            if (e.y == kC || !ctab) {
                // rows past the end of a batch row are clipped by the tensor store
                if (leader) {
                    tc::tma_store_4d(&maps.out, stg, 0, h, e.x, ctab ? 0 : bh / H);
                    tc::bulk_commit();
                }
            } else {
                // a packed sequence's short last chunk: the rows after it belong to the next
                // sequence, so only its own rows are written (16-byte plain stores)
                const int o = tid - 384;
                for (int x = o; x < e.y * 16; x += 128) {
                    const int r = x >> 4, col = x & 15;
                    if (e.x + r < T_len) {
                        const uint4 val = *reinterpret_cast<const uint4*>(stg + r * 256 + col * 16);
                        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(out) +
                                                  ((size_t)(e.x + r) * H + h) * (kDV * 2) + col * 16) = val;
                    }
                }
                // the staging tile is read before the next item rewrites it
                tc::bar_named(1, 128);
            }
            if constexpr (kSeg) {
                it.next();
            } else if (++c == nc) {
                c = 0;
                bh += hstride;
                if (u + 1 < U) {
                    nc = units_chunks(bh);
                    if (ctab) otab = ctab + (size_t)(bh / H) * NT;
                }
            }
        }
        if (leader) tc::bulk_wait_all();
    }
    tc::tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) record_status(kStatusStateWait);
}

__device__ __forceinline__ uint8_t* aligned_smem(uint8_t* raw) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

// Tensor Memory belongs to the kernel, not to a role: one allocation of all 512 columns (one CTA
// per SM), after which the CTA gives up its permit to allocate, so a CTA that changes role keeps
// the same columns.
__device__ __forceinline__ uint32_t kernel_tmem_alloc(uint32_t* slot) {
    if ((threadIdx.x >> 5) == 0) {
        tc::tmem_alloc(slot, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    return *slot;
}
__device__ __forceinline__ void kernel_tmem_free(uint32_t tmem) {
    tc::tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) tc::tmem_dealloc(tmem, 512);
}

// Factor kernel alone: persistent over every chunk-head (chunk-major over all heads).
template <bool kLogits>
__global__ void __launch_bounds__(512, 1)
ckda_tc_intra(const __grid_constant__ TcMaps maps, const void* __restrict__ alpha,
              const float* __restrict__ beta, uint8_t* __restrict__ ws, int* __restrict__ flags,
              PackedTabs pt, int T_len, int H, int NT, int n_items, WorkOrder wo,
              int l2norm, RopeParams rp, long long pos_offset) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_slot;
    const uint32_t tmem = kernel_tmem_alloc(&tmem_slot);
    const ItemSeq seq{(int)blockIdx.x, (int)gridDim.x, 1 << 30, 0, 1, n_items};
    intra_role<kLogits>(aligned_smem(smem_raw), maps, alpha, beta, ws, flags, pt, T_len, H, NT, wo,
                        seq, l2norm, rp, pos_offset, tmem);
    kernel_tmem_free(tmem);
}

// State pass alone, after the factor kernel: heads blockIdx.x, blockIdx.x + gridDim.x, ...
__global__ void __launch_bounds__(512, 1)
ckda_tc_state(const __grid_constant__ TcMaps maps, const uint8_t* __restrict__ ws,
              const int* __restrict__ flags, PackedTabs pt,
              const float* __restrict__ h0, __nv_bfloat16* __restrict__ out,
              float* __restrict__ hT, int T_len, int H, int NT, int BH, float scale) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_slot;
    const uint32_t tmem = kernel_tmem_alloc(&tmem_slot);
    state_role<false>(aligned_smem(smem_raw), maps, ws, flags, pt, h0, out, hT, T_len, H, NT, BH,
                      scale, blockIdx.x, gridDim.x, tmem, SegArgs{});
    kernel_tmem_free(tmem);
}

// Both at once (cooperative launch, every CTA resident).  Every CTA first takes `lead` rounds of
// factor items (item blockIdx.x + r gridDim.x, r < lead); then CTAs 0 .. n_state - 1 carry the
// chains of heads blockIdx.x + k n_state, and the others take the remaining items in turn.  The
// items run in head groups of n_state, chunk-major inside a group, so the chains of a group run
// while the group's chunks are produced.  A chain CTA waits only on flags that factor work
// raises, and factor work never waits on a chain, so every wait ends.
template <bool kLogits>
__global__ void __launch_bounds__(512, 1)
ckda_tc_fused(const __grid_constant__ TcMaps maps, const void* __restrict__ alpha,
              const float* __restrict__ beta, uint8_t* __restrict__ ws, int* __restrict__ flags,
              PackedTabs pt, const float* __restrict__ h0,
              __nv_bfloat16* __restrict__ out, float* __restrict__ hT, int T_len, int H, int NT,
              int BH, int n_items, int n_state, int lead, WorkOrder wo, int l2norm, RopeParams rp,
              long long pos_offset, float scale) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_slot;
    uint8_t* sm = aligned_smem(smem_raw);
    const uint32_t tmem = kernel_tmem_alloc(&tmem_slot);
    const int total = n_items, b = blockIdx.x, nall = gridDim.x, nf = nall - n_state;
    const bool chain = b < n_state;
    // the leading rounds, then (factor CTAs) every nf-th of the remaining items
    const ItemSeq seq{b, nall, lead, chain ? total : lead * nall + (b - n_state), chain ? 1 : nf, total};
    if (seq.at(0) >= 0)
        intra_role<kLogits>(sm, maps, alpha, beta, ws, flags, pt, T_len, H, NT, wo, seq, l2norm,
                            rp, pos_offset, tmem);
    if (chain)
        state_role<false>(sm, maps, ws, flags, pt, h0, out, hT, T_len, H, NT, BH, scale, b, n_state,
                          tmem, SegArgs{});
    kernel_tmem_free(tmem);
}

// A pass over segment units (after the factor kernel): units blockIdx.x, blockIdx.x + gridDim.x, ...
__global__ void __launch_bounds__(512, 1)
ckda_tc_seg(const __grid_constant__ TcMaps maps, const uint8_t* __restrict__ ws,
            const int* __restrict__ flags, const float* __restrict__ h0,
            __nv_bfloat16* __restrict__ out, float* __restrict__ hT, int T_len, int H, int NT,
            int BH, float scale, SegArgs sa) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_slot;
    const uint32_t tmem = kernel_tmem_alloc(&tmem_slot);
    state_role<true>(aligned_smem(smem_raw), maps, ws, flags, PackedTabs{nullptr, nullptr, nullptr},
                     h0, out, hT, T_len, H, NT, BH, scale, blockIdx.x, gridDim.x, tmem, sa);
    kernel_tmem_free(tmem);
}

// The scan over the segments of one head unit, 8 state columns per CTA (grid BH x 16), in fp32 on
// CUDA cores: S_0 = h0 (or zero), S_1 = E_0, S_{s+1} = F_s S_s + E_s for 0 < s < P - 1.  F_{s+1}
// is copied into shared memory (rows 132 floats apart) while step s runs; thread (row r, column
// group) reads its row of F_s in 16-byte pieces (eight consecutive rows of a quarter warp fall on
// distinct bank groups) and forms 4 columns.
constexpr int kScanCols = 8, kScanLd = kDK + 4, kScanThreads = 256;
constexpr size_t kScanSmem = sizeof(float) * (2 * (size_t)kDK * kScanLd + (size_t)kDK * kScanCols);
__device__ __forceinline__ void scan_load_f(float* dst, const float* F) {
    for (int i = threadIdx.x; i < kDK * kDK / 4; i += kScanThreads) {
        const int r = i / (kDK / 4), k4 = 4 * (i % (kDK / 4));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                     ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst + r * kScanLd + k4))),
                     "l"(F + (size_t)r * kDK + k4) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__global__ void __launch_bounds__(kScanThreads)
ckda_seg_scan(const float* __restrict__ h0, SegArgs sa) {
    extern __shared__ __align__(16) float scan_sm[];
    float* sF = scan_sm;                            // F_s, two buffers [128][132]
    float* sS = scan_sm + 2 * kDK * kScanLd;        // S_s columns [128][8]
    const int bh = blockIdx.x, n0 = blockIdx.y * kScanCols, tid = threadIdx.x;
    const size_t st = (size_t)kDK * kDV, base = (size_t)bh * sa.P;
    float* segS = const_cast<float*>(sa.segS);
    tc::grid_dependency_wait();   // the summary pass is complete (programmatic launch)
    // F_s goes to buffer s & 1
    if (sa.P > 2) scan_load_f(sF + kDK * kScanLd, sa.segF + (base + 1) * st);
    for (int e = tid; e < kDK * kScanCols; e += kScanThreads) {
        const size_t o = (size_t)(e / kScanCols) * kDV + n0 + e % kScanCols;
        segS[base * st + o] = h0 ? h0[(size_t)bh * st + o] : 0.f;
        const float s1 = sa.segE[base * st + o];
        sS[e] = s1;
        segS[(base + 1) * st + o] = s1;
    }
    const int r = tid >> 1, cg = 4 * (tid & 1);
    // this thread's part of E_s, loaded one step ahead
    auto load_e = [&](int s) {
        return *reinterpret_cast<const float4*>(sa.segE + (base + s) * st + (size_t)r * kDV + n0 + cg);
    };
    float4 e_next = sa.P > 2 ? load_e(1) : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 1; s + 1 < sa.P; ++s) {
        const float4 e4 = e_next;
        if (s + 2 < sa.P) e_next = load_e(s + 1);
        if (s + 2 < sa.P) {
            scan_load_f(sF + ((s + 1) & 1) * kDK * kScanLd, sa.segF + (base + s + 1) * st);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();   // F_s landed (every thread's copies) and S_s written
        const float4* Fr = reinterpret_cast<const float4*>(sF + (s & 1) * kDK * kScanLd + r * kScanLd);
        float a0 = e4.x, a1 = e4.y, a2 = e4.z, a3 = e4.w;
#pragma unroll 8
        for (int k4 = 0; k4 < kDK / 4; ++k4) {
            const float4 f = Fr[k4];
            const float fk[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const float4 sv = *reinterpret_cast<const float4*>(sS + (4 * k4 + kk) * kScanCols + cg);
                a0 += fk[kk] * sv.x;
                a1 += fk[kk] * sv.y;
                a2 += fk[kk] * sv.z;
                a3 += fk[kk] * sv.w;
            }
        }
        __syncthreads();   // every thread has read S_s and F_s
        *reinterpret_cast<float4*>(sS + r * kScanCols + cg) = make_float4(a0, a1, a2, a3);
        *reinterpret_cast<float4*>(segS + (base + s + 1) * st + (size_t)r * kDV + n0 + cg) =
            make_float4(a0, a1, a2, a3);
    }
}

// Packed sequences: the tables and the ready flags of one call (one CTA of 1024 threads).
//  1. chunk table: sequences are taken 1024 at a time; a block-wide scan of their chunk counts
//     gives each one its first chunk in the global order, and lane l's chunk j is global chunk
//     cbase[l] + j.  Slots past a lane's count get a harmless entry (never read).
//  2. item table: head unit u = lane * H + h has lane_cnt[lane] chunks; units form groups of
//     `group` (the chain CTAs of the launch), and inside a group the items run chunk-major over
//     the units that have that chunk.  Item (u, c) sits at base(group) + sum over the group's
//     units of min(count, c) + the number of the group's units before u that have chunk c.
// If the device offsets do not match the plan (the two copies of cu_seqlens differ), every chunk
// entry becomes an empty chunk of sequence 0 and the error word is set, so that no later access
// leaves the caller's arrays.
constexpr int kPrepThreads = 1024;
__global__ void __launch_bounds__(kPrepThreads)
ckda_varlen_prep(const int* __restrict__ cu, int n_seqs, int T_total, const LanePlan lp, int H,
                 int group, int4* __restrict__ ctab, int* __restrict__ lane_cnt,
                 int2* __restrict__ itab, int* __restrict__ flags, int n_flags) {
    __shared__ int warp_sum[32];
    __shared__ int s_bad;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto cnt = [&](int l) { return lp.cbase[l + 1] - lp.cbase[l]; };
    for (int i = tid; i < n_flags; i += kPrepThreads) flags[i] = 0;
    if (tid < lp.P) lane_cnt[tid] = cnt(tid);
    if (tid == 0) s_bad = (cu[0] != 0 || cu[n_seqs] != T_total) ? 1 : 0;
    __syncthreads();
    // 1. chunk table
    int base = 0;   // chunks of the sequences before this tile
    for (int s0 = 0; s0 < n_seqs; s0 += kPrepThreads) {
        const int sq = s0 + tid;
        int len = 0;
        if (sq < n_seqs) {
            len = cu[sq + 1] - cu[sq];
            if (len < 0) {
                s_bad = 1;
                len = 0;
            }
        }
        const int nch = (len + kC - 1) / kC;
        // inclusive scan of nch over the block
        int x = nch;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, d);
            if (lane >= d) x += y;
        }
        if (lane == 31) warp_sum[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sum[lane];
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, d);
                if (lane >= d) w += y;
            }
            warp_sum[lane] = w;   // inclusive over warps
        }
        __syncthreads();
        const int first = base + (warp ? warp_sum[warp - 1] : 0) + x - nch;
        const int tile_total = warp_sum[31];
        if (nch > 0) {
            int l = 0;   // the lane of sequence sq
            while (l + 1 < lp.P && lp.seq0[l + 1] <= sq) ++l;
            for (int j = 0; j < nch; ++j) {
                const int jl = first + j - lp.cbase[l];
                if (jl >= 0 && jl < cnt(l))
                    ctab[(size_t)l * lp.NTL + jl] = make_int4(cu[sq] + j * kC, min(kC, len - j * kC),
                                                              sq, j | (j == nch - 1 ? kLastChunk : 0));
                else
                    s_bad = 1;
            }
        }
        base += tile_total;
        __syncthreads();   // warp_sum is rewritten by the next tile
    }
    for (int x = tid; x < lp.P * lp.NTL; x += kPrepThreads) {
        const int l = x / lp.NTL;
        if (x - l * lp.NTL >= cnt(l)) ctab[x] = make_int4(0, 0, min(lp.seq0[l], n_seqs - 1), 1);
    }
    __syncthreads();
    if (base != lp.total) s_bad = 1;
    __syncthreads();
    if (s_bad) {
        for (int x = tid; x < lp.P * lp.NTL; x += kPrepThreads) ctab[x] = make_int4(0, 0, 0, 0);
        if (tid == 0) record_status(kStatusPackedOffsets);
    }
    // 2. item table
    const int BH = lp.P * H;
    for (int u = tid; u < BH; u += kPrepThreads) {
        const int l = u / H, n_u = cnt(l);
        const int g0 = u - u % group, g1 = min(BH, g0 + group);
        const int la = g0 / H, lb = (g1 - 1) / H;
        const long long gbase = (long long)H * lp.cbase[la] + (long long)(g0 - la * H) * cnt(la);
        const int own = u - max(g0, l * H);   // units of u's lane ahead of u in the group
        long long S = 0;                      // sum over the group's units of min(count, c)
        for (int c = 0; c < n_u; ++c) {
            int rank = own, ng = 0;
            for (int l2 = la; l2 <= lb; ++l2) {
                const int m = min(g1, (l2 + 1) * H) - max(g0, l2 * H);   // the lane's units in the group
                const int on = cnt(l2) > c ? m : 0;
                ng += on;
                if (l2 < l) rank += on;
            }
            itab[gbase + S + rank] = make_int2(u, c);
            S += ng;
        }
    }
}

// Empty packed sequences: hT = h0 (or zero) for the listed sequences, one CTA per sequence.
constexpr int kMaxEmptyList = 1024;
struct EmptyList {
    int n;
    int seq[kMaxEmptyList];
};
__global__ void __launch_bounds__(256)
ckda_varlen_empty(const __grid_constant__ EmptyList list, const float* __restrict__ h0,
                  float* __restrict__ hT, int H) {
    const size_t per = (size_t)H * kDK * kDV;
    const size_t o = (size_t)list.seq[blockIdx.x] * per;
    for (size_t i = threadIdx.x * 4; i < per; i += 256 * 4) {
        const float4 x = h0 ? *reinterpret_cast<const float4*>(h0 + o + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(hT + o + i) = x;
    }
}

}  // namespace

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// A [B][T][H][C] array as a 4-D tensor {C, H, T, B}; box = `box_c` channels of 64 tokens of one
// (batch, head).  Tokens past T read as zeros.
static bool encode_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int C,
                int box_c, int H, int T_len, int B, CUtensorMapSwizzle sw) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)H, (cuuint64_t)T_len, (cuuint64_t)B};
    const cuuint64_t row = (cuuint64_t)C * esize;
    const cuuint64_t strides[3] = {row, row * H, row * H * T_len};
    const cuuint32_t box[4] = {(cuuint32_t)box_c, 1, (cuuint32_t)kC, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Workspace: the images of n = heads x chunks chunk-heads, their ready flags, and (packed
// sequences) the chunk table of `ntab` entries.
// Workspace: the images of n = units x NT chunk slots and their ready flags; for packed sequences
// then the chunk table (lanes x NT entries), the lane counts and the item table.
static size_t ctab_offset(size_t n) { return flags_offset(n) + ((n * 4 + 255) & ~(size_t)255); }

size_t chunk_tc_workspace_bytes(int B, int T_len, int H) {
    const size_t nt = (size_t)(T_len + kC - 1) / kC;
    return ctab_offset((size_t)B * H * nt);
}

long long packed_chunks(const int* cu_host, int n_seqs) {
    long long nc = 0;
    for (int s = 0; s < n_seqs; ++s) nc += (cu_host[s + 1] - cu_host[s] + kC - 1) / kC;
    return nc;
}

struct PackedLayout {
    size_t images, ctab, lane_cnt, itab, bytes;   // byte offsets into the workspace, and its size
};
static PackedLayout packed_layout(const LanePlan& lp, int H) {
    PackedLayout w;
    const size_t slots = (size_t)lp.P * H * lp.NTL;
    w.images = 0;
    w.ctab = ctab_offset(slots);
    w.lane_cnt = w.ctab + (size_t)lp.P * lp.NTL * sizeof(int4);
    w.itab = w.lane_cnt + (((size_t)lp.P * 4 + 15) & ~(size_t)15);
    w.bytes = w.itab + (size_t)H * lp.total * sizeof(int2);
    return w;
}

size_t chunk_tc_workspace_bytes_packed(const int* cu_host, int n_seqs, int H) {
    return packed_layout(plan_lanes(cu_host, n_seqs, kC), H).bytes;
}

// Split of the fused launch: `n_state` chain CTAs, and `lead` leading rounds of factor items that
// every CTA (chain CTAs included) takes before the chains start.  Model (SM cycles, measured on
// B200): a round of factor items takes t_i = 19000 on every CTA in step, an item is flagged ready
// about 1.5 rounds after the round it starts in, and a chain step takes t_c = 2200.  With s chain
// CTAs the heads form groups of s, produced one after the other (chunk-major inside a group);
// chain CTA 0 carries the first head of every group in turn, so it finishes last.  Its head in
// group g cannot end before the previous head plus NT steps, before that head's first chunk plus
// NT steps, or before its last chunk plus one step (and no chain starts before the leading rounds
// are done).  The split minimises the later of that end and the end of the factor work (the
// larger s and the smaller lead on ties).
void chunk_tc_plan(int BH, int NT, long long n_items, int nsm, int* n_state, int* lead,
                   double* t_model) {
    struct Entry {
        int BH, NT;
        long long n_items;
        int nsm, s, lead;
        double t;
    };
    static std::mutex m;
    static Entry cache[16];
    static int n_cached = 0;
    {
        std::lock_guard<std::mutex> g(m);
        for (int e = 0; e < n_cached; ++e)
            if (cache[e].BH == BH && cache[e].NT == NT && cache[e].n_items == n_items &&
                cache[e].nsm == nsm) {
                *n_state = cache[e].s;
                *lead = cache[e].lead;
                if (t_model) *t_model = cache[e].t;
                return;
            }
    }
    const double ti = 19000.0, tc = 2200.0, lag = 1.5;
    // items: BH x NT, or fewer for packed sequences, whose lanes hold up to NT chunks each
    const long long total = n_items;
    const double per_unit = (double)n_items / BH;
    const int smax = BH < nsm - 1 ? BH : nsm - 1;
    const int lmax = (int)((total + nsm - 1) / nsm) < 8 ? (int)((total + nsm - 1) / nsm) : 8;
    int best_s = 1, best_l = 0;
    double best_t = 1e300;
    for (int s = 1; s <= smax; ++s) {
        const long long nf = nsm - s;
        for (int l = 0; l <= lmax; ++l) {
            const long long pre = (long long)l * nsm < total ? (long long)l * nsm : total;
            const long long rest = total - pre;
            auto round_of = [&](long long i) {
                return i < pre ? (double)(i / nsm) : (double)l + (double)((i - pre) / nf);
            };
            const double factor_end =
                ((double)((pre + nsm - 1) / nsm) + (double)((rest + nf - 1) / nf)) * ti;
            double end = (double)l * ti;
            for (int g = 0; (long long)g * s < BH; ++g) {
                const long long sg = BH - (long long)g * s < s ? BH - (long long)g * s : s;
                const long long first = (long long)((double)g * s * per_unit);
                long long last_item = first + (long long)(NT - 1) * sg;
                if (last_item > total - 1) last_item = total - 1;
                const double t_first = (round_of(first) + lag) * ti;
                const double t_last = (round_of(last_item) + lag) * ti;
                double e = end + NT * tc;
                if (t_first + NT * tc > e) e = t_first + NT * tc;
                if (t_last + tc > e) e = t_last + tc;
                end = e;
            }
            const double t = end > factor_end ? end : factor_end;
            if (t < best_t - 1.0 || (t <= best_t + 1.0 && s > best_s)) {
                best_t = t;
                best_s = s;
                best_l = l;
            }
        }
    }
    *n_state = best_s;
    *lead = best_l;
    if (t_model) *t_model = best_t;
    std::lock_guard<std::mutex> g(m);
    if (n_cached < 16) cache[n_cached++] = Entry{BH, NT, n_items, nsm, best_s, best_l, best_t};
}

// Segments of the segment-parallel pass: L = ceil(NT / P) chunks each, and as many segments as
// that needs (none empty).
static void seg_shape(int NT, int P, int* Pe, int* L) {
    const int l = (NT + P - 1) / P;
    *L = l;
    *Pe = (NT + l - 1) / l;
}

size_t chunk_tc_seg_workspace_bytes(int B, int T_len, int H, int segments) {
    const int NT = (T_len + kC - 1) / kC;
    int P = 1, L = NT;
    if (segments > 1) seg_shape(NT, segments, &P, &L);
    const size_t base = chunk_tc_workspace_bytes(B, T_len, H);
    if (P < 2) return base;
    return ((base + 255) & ~(size_t)255) + 3 * (size_t)B * H * P * kDK * kDV * sizeof(float);
}

// Segment count for the segment-parallel pass, from the same cycle model as chunk_tc_plan: the
// factor kernel alone (rounds of t_i on all SMs), the summary pass (end-state and transition
// chains, rounds of L steps of t_c), the scan (t_s per segment), the pass with outputs (rounds of
// L steps) and t_g for the flag reset and the four launches (t_s and t_g fitted to B200 timings
// of one sequence of 65536 tokens on 2 heads).  1 when no segment count beats the single fused
// launch.
int chunk_tc_seg_plan(int BH, int NT, int nsm) {
    const double ti = 19000.0, tc = 2200.0, ts = 5000.0, tg = 35000.0;
    if (BH < 1 || NT < 4 || nsm < 2) return 1;
    int n_state = 1, lead = 0;
    double fused = 0.0;
    chunk_tc_plan(BH, NT, (long long)BH * NT, nsm, &n_state, &lead, &fused);
    const double factor = (double)(((long long)BH * NT + nsm - 1) / nsm) * ti;
    int best = 1;
    double best_t = fused;
    for (int p = 2; p <= NT && p <= 1024; ++p) {
        int P, L;
        seg_shape(NT, p, &P, &L);
        if (P != p) continue;
        const long long nsum = (long long)BH * (P - 1) + (long long)BH * (P - 2);
        const double t = factor + (double)((nsum + nsm - 1) / nsm) * L * tc + (P - 2) * ts +
                         (double)(((long long)BH * P + nsm - 1) / nsm) * L * tc + tg;
        if (t < best_t) {
            best_t = t;
            best = P;
        }
    }
    return best;
}

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const void* alpha,
                            const float* beta, const float* h0, void* out, float* hT, int B,
                            int T_len, int H, int G, int l2norm, const RopeParams& rp, float scale,
                            long long pos_offset, int gate_logits, void* workspace, int stages,
                            const PackedSeqs& pk, cudaStream_t stream) {
    auto intra = gate_logits ? ckda_tc_intra<true> : ckda_tc_intra<false>;
    auto fused = gate_logits ? ckda_tc_fused<true> : ckda_tc_fused<false>;
    cudaError_t e = cudaFuncSetAttribute(intra, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ckda_tc_state, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SS_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fused, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FUSED_BYTES);
    if (e != cudaSuccess) return e;
    // packed sequences: one token axis (batch 1); the sequences are dealt to lanes that stand in
    // for batch rows, and a unit's chain walks through its lane's sequences, starting again from
    // h0 at each one
    const bool packed = pk.cu != nullptr;
    LanePlan lp;
    if (packed) lp = plan_lanes(pk.cu_host, pk.n, kC);
    const int NT = packed ? lp.NTL : (T_len + kC - 1) / kC;
    const int BH = packed ? lp.P * H : B * H;
    const int Bm = packed ? 1 : B;
    const int total = NT * BH;                                 // chunk slots (images, flags)
    const int n_items = packed ? H * lp.total : total;         // chunk-heads to produce
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int* flags = reinterpret_cast<int*>(ws + flags_offset((size_t)total));
    PackedTabs pt{nullptr, nullptr, nullptr};
    if (packed) {
        const PackedLayout pl = packed_layout(lp, H);
        pt.ctab = reinterpret_cast<const int4*>(ws + pl.ctab);
        pt.lane_cnt = reinterpret_cast<const int*>(ws + pl.lane_cnt);
        pt.itab = reinterpret_cast<const int2*>(ws + pl.itab);
    }
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (stages == 0 && nsm < 2) stages = 3;
    int n_state = 1, lead = 0;
    if (stages == 0 && n_items > 0) chunk_tc_plan(BH, NT, n_items, nsm, &n_state, &lead, nullptr);
    if (packed && stages != 2) {
        if (hT) {
            // empty sequences keep their initial state
            EmptyList list;
            list.n = 0;
            for (int s = 0; s <= pk.n; ++s) {
                if (s < pk.n && pk.cu_host[s + 1] == pk.cu_host[s]) list.seq[list.n++] = s;
                if (list.n == kMaxEmptyList || (s == pk.n && list.n > 0)) {
                    ckda_varlen_empty<<<list.n, 256, 0, stream>>>(list, h0, hT, H);
                    if ((e = cudaGetLastError()) != cudaSuccess) return e;
                    list.n = 0;
                }
            }
        }
        if (n_items == 0) return cudaSuccess;
        // the chunk and item tables (items grouped as the launch takes them: by chain CTA for the
        // fused kernel, all units at once for the factor kernel alone), every ready flag at zero
        ckda_varlen_prep<<<1, kPrepThreads, 0, stream>>>(
            pk.cu, pk.n, T_len, lp, H, stages == 0 ? n_state : BH, const_cast<int4*>(pt.ctab),
            const_cast<int*>(pt.lane_cnt), const_cast<int2*>(pt.itab), flags, total);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (n_items == 0) return cudaSuccess;
    __nv_bfloat16* outb = static_cast<__nv_bfloat16*>(out);
    TcMaps maps;
    if (!encode_map(&maps.out, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDV, kDV, H, T_len, Bm,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (stages != 2) {
        // q and k carry H / G heads (value head h reads q/k head h / G)
        if (!encode_map(&maps.q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDK, kDK, H / G, T_len, Bm,
                        CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode_map(&maps.k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDK, kDK, H / G, T_len, Bm,
                        CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode_map(&maps.v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDV, 64, H, T_len, Bm,
                        CU_TENSOR_MAP_SWIZZLE_128B) ||
            !(gate_logits ? encode_map(&maps.alpha, alpha, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDK,
                                       kDK, H, T_len, Bm, CU_TENSOR_MAP_SWIZZLE_NONE)
                          : encode_map(&maps.alpha, alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kDK,
                                       kDK, H, T_len, Bm, CU_TENSOR_MAP_SWIZZLE_NONE)))
            return cudaErrorInvalidValue;
        // every ready flag starts at zero; the factor role raises them (packed sequences: the
        // table kernel above cleared them)
        if (!packed) {
            e = cudaMemsetAsync(flags, 0, (size_t)total * 4, stream);
            if (e != cudaSuccess) return e;
        }
    }
    if (stages == 0) {
        // one cooperative launch: the runtime makes every CTA resident at once, which the chain
        // CTAs (waiting on flags the factor CTAs raise) rely on
        // every CTA takes part in the leading rounds; afterwards only the factor CTAs take items
        const int n_intra = nsm - n_state;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(n_state + n_intra));
        cfg.blockDim = dim3(512);
        cfg.dynamicSmemBytes = FUSED_BYTES;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, fused, maps, alpha, beta, ws, flags, pt, h0, outb, hT,
                                  T_len, H, NT, BH, n_items, n_state, lead,
                                  make_work_order(NT, BH, H, n_state, G), l2norm, rp, pos_offset,
                                  scale);
    }
    // two kernels in sequence (profiling aid).  The factor kernel follows the flag reset in plain
    // stream order; the state kernel uses programmatic dependent launch (its set-up overlaps the
    // factor kernel's tail, and griddepcontrol.wait holds it back before it reads the workspace)
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (stages & 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(n_items < nsm ? n_items : nsm));
        cfg.blockDim = dim3(512);
        cfg.dynamicSmemBytes = S_BYTES;
        cfg.stream = stream;
        e = cudaLaunchKernelEx(&cfg, intra, maps, alpha, beta, ws, flags, pt, T_len, H, NT, n_items,
                               make_work_order(NT, BH, H, BH, G), l2norm, rp, pos_offset);
        if (e != cudaSuccess) return e;
    }
    if (stages & 2) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)BH);
        cfg.blockDim = dim3(512);
        cfg.dynamicSmemBytes = SS_BYTES;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, ckda_tc_state, maps, static_cast<const uint8_t*>(ws),
                               static_cast<const int*>(flags), pt, h0, outb, hT, T_len, H, NT, BH,
                               scale);
    }
    return e;
}

// The forward with the segment-parallel pass (batched sequences only): the factor kernel, the
// summary pass, the scan, and the pass with outputs, in stream order.
cudaError_t launch_chunk_tc_seg(const void* q, const void* k, const void* v, const void* alpha,
                                const float* beta, const float* h0, void* out, float* hT, int B,
                                int T_len, int H, int G, int l2norm, const RopeParams& rp,
                                float scale, long long pos_offset, int gate_logits,
                                void* workspace, int segments, cudaStream_t stream) {
    const int NT = (T_len + kC - 1) / kC, BH = B * H;
    const PackedSeqs none{nullptr, nullptr, 0};
    int P = 1, L = NT;
    if (segments > 1) seg_shape(NT, segments, &P, &L);
    if (P < 2)
        return launch_chunk_tc(q, k, v, alpha, beta, h0, out, hT, B, T_len, H, G, l2norm, rp, scale,
                               pos_offset, gate_logits, workspace, 0, none, stream);
    // the factor kernel (with the reset of the ready flags)
    cudaError_t e = launch_chunk_tc(q, k, v, alpha, beta, h0, out, hT, B, T_len, H, G, l2norm, rp,
                                    scale, pos_offset, gate_logits, workspace, 1, none, stream);
    if (e != cudaSuccess) return e;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int* flags = reinterpret_cast<const int*>(ws + flags_offset((size_t)BH * NT));
    float* seg = reinterpret_cast<float*>(
        ws + ((chunk_tc_workspace_bytes(B, T_len, H) + 255) & ~(size_t)255));
    const size_t arr = (size_t)BH * P * kDK * kDV;
    SegArgs sa{P, L, 1, seg, seg + arr, seg + 2 * arr};
    TcMaps maps;
    if (!encode_map(&maps.out, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDV, kDV, H, T_len, B,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(ckda_tc_seg, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SS_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ckda_seg_scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kScanSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    __nv_bfloat16* outb = static_cast<__nv_bfloat16*>(out);
    // programmatic dependent launches: each kernel's set-up overlaps the previous one's tail, and
    // griddepcontrol.wait holds it back before it reads what that kernel wrote
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(512);
    cfg.dynamicSmemBytes = SS_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int nsum = seg_units(sa, BH);
    cfg.gridDim = dim3((unsigned)(nsum < nsm ? nsum : nsm));
    e = cudaLaunchKernelEx(&cfg, ckda_tc_seg, maps, static_cast<const uint8_t*>(ws), flags, h0,
                           outb, hT, T_len, H, NT, BH, scale, sa);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t scfg = cfg;
    scfg.gridDim = dim3((unsigned)BH, kDV / kScanCols);
    scfg.blockDim = dim3(kScanThreads);
    scfg.dynamicSmemBytes = kScanSmem;
    e = cudaLaunchKernelEx(&scfg, ckda_seg_scan, h0, sa);
    if (e != cudaSuccess) return e;
    sa.summary = 0;
    const int npass = BH * P;
    cfg.gridDim = dim3((unsigned)(npass < nsm ? npass : nsm));
    return cudaLaunchKernelEx(&cfg, ckda_tc_seg, maps, static_cast<const uint8_t*>(ws), flags, h0,
                              outb, hT, T_len, H, NT, BH, scale, sa);
}

// Read the status word on the current device (after `stream` has finished) and clear it.
cudaError_t device_status_take(cudaStream_t stream, int* code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_tc_error, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && v != 0) {
        static const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_tc_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                                    stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    }
    *code = v;
    return e;
}

// Bound of one wait of the state role on the current device (0: the default).
cudaError_t set_wait_limit_ns(unsigned long long ns) {
    const unsigned long long v = ns ? ns : kDefaultWaitNs;
    return cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v));
}

}  // namespace ckda
