// chunk_records.cuh -- the per-chunk factor records of the CUDA-core chunked passes and the
// warp-level tensor-core tiles they use (the backward, chunk_bwd.cu, and the CUDA-core forward,
// chunk_simt.cu).  Chunks of 16 tokens; the factors are those of simt_chunk.cuh.
#pragma once

#include "simt_chunk.cuh"

namespace ckda {

namespace {

using simt::Factors;
using simt::kThreads;

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

// ---- warp-level tensor-core tiles with fp32-grade products ------------------------------------
// mma.sync m16n8k8 with tf32 operands, each operand split into a tf32 head and a tf32 tail
// (x = hi + lo: hi is x with its 13 low mantissa bits cleared, lo the remainder x - hi, exact in
// fp32, with its own 13 low bits cleared; each cut loses under 2^-10 of what it cuts):
// a b = a_hi b_hi + a_hi b_lo + a_lo b_hi up to a relative 3 * 2^-20, i.e. the product of two
// fp32 values to about fp32 precision ("3xTF32").  The cuts are integer masks on the full-rate
// pipes.  Fragment layout
// (PTX ISA, mma.m16n8k8 .tf32), g = lane / 4, t = lane % 4: A a0 = A[g][t], a1 = A[g+8][t],
// a2 = A[g][t+4], a3 = A[g+8][t+4]; B b0 = B[t][g], b1 = B[t+4][g]; D d0 = D[g][2t],
// d1 = D[g][2t+1], d2 = D[g+8][2t], d3 = D[g+8][2t+1].
constexpr uint32_t kTf32Mask = 0xffffe000u;   // sign, exponent and the 10 tf32 mantissa bits
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = __float_as_uint(x) & kTf32Mask;
    lo = __float_as_uint(x - __uint_as_float(hi)) & kTf32Mask;
}
__device__ __forceinline__ void mma_tf32(float c[4], const uint32_t a[4], const uint32_t b[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// c (+)= A[16 x K] B[K x 8], A(m, k) and B(k, n) read through the accessors
template <int K, typename FA, typename FB>
__device__ __forceinline__ void mma3_tile(float c[4], FA A, FB B, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        uint32_t ah[4], al[4], bh[2], bl[2];
        split_tf32(A(g, k0 + t), ah[0], al[0]);
        split_tf32(A(g + 8, k0 + t), ah[1], al[1]);
        split_tf32(A(g, k0 + t + 4), ah[2], al[2]);
        split_tf32(A(g + 8, k0 + t + 4), ah[3], al[3]);
        split_tf32(B(k0 + t, g), bh[0], bl[0]);
        split_tf32(B(k0 + t + 4, g), bh[1], bl[1]);
        mma_tf32(c, al, bh);
        mma_tf32(c, ah, bl);
        mma_tf32(c, ah, bh);
    }
}
// D fragment (times s) into rows ld floats apart, columns col0 ..
__device__ __forceinline__ void st_frag(float* d, int ld, int col0, const float c[4], float s,
                                        int lane) {
    const int g = lane >> 2, t = lane & 3;
    d[g * ld + col0 + 2 * t] = s * c[0];
    d[g * ld + col0 + 2 * t + 1] = s * c[1];
    d[(g + 8) * ld + col0 + 2 * t] = s * c[2];
    d[(g + 8) * ld + col0 + 2 * t + 1] = s * c[3];
}

// ---- A, M, T and W of a 16-token chunk on the warp tiles ------------------------------------------
// When every channel's decay over the chunk stays >= 2^-118 (L_C >= -118), each gate ratio
// R_rj = g_r / g_j (g = exp2(L) = |gamma|) factors into g_r and 1/g_j, both inside the fp32 range,
// and the per-channel sums become dense products:
//   A = diag(beta) strict_lower(K_gamma (K / g)^T),  M = lower(Q_gamma (K / g)^T),
//   W = T diag(beta) K_gamma,   with K_gamma = g k', Q_gamma = g q', K / g = k' / g.
// The products masked out (j > r) stay finite: g_r / g_j <= 2^118 there.  T is solved as in
// chunk_products.  On return f.q holds Q_gamma, f.k holds K / g and f.L holds K_gamma, and the
// result is true; otherwise (a chunk whose decay falls below 2^-118 somewhere, exact zeros
// included) chunk_products runs unchanged on the exact ratios exp2(L_r - L_j) and the result is
// false.  P (nullable, [C][C]) receives A before the row scaling by beta.  Ends with a barrier.
template <int DK, int C>
__device__ __forceinline__ bool chunk_products_tiles(const Factors<DK, C>& f, float* P) {
    static_assert(C == 16, "one 16-row warp tile per chunk");
    constexpr int LD = Factors<DK, C>::LD;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool safe = __syncthreads_and(tid >= DK || f.LC[tid] >= -118.f) != 0;
    if (!safe) {
        simt::chunk_products<DK, C>(f, P);
        return false;
    }
    for (int e = tid; e < C * DK; e += kThreads) {
        const int r = e / DK, c = e % DK, o = r * LD + c;
        const float L = f.L[o], g = exp2f(L), kp = f.k[o];
        f.L[o] = g * kp;                    // K_gamma
        f.q[o] = g * f.q[o];                // Q_gamma
        f.k[o] = kp * exp2f(-L);            // K / g
    }
    __syncthreads();
    // warps 0-1: A (8-column tiles 0, 1), warps 2-3: M
    if (warp < 4) {
        const int nt = warp & 1;
        const float* X = warp < 2 ? f.L : f.q;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        mma3_tile<DK>(c, [&](int m, int kk) { return X[m * LD + kk]; },
                      [&](int kk, int n) { return f.k[(8 * nt + n) * LD + kk]; }, lane);
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = g + 8 * (i >> 1), j = 8 * nt + 2 * t + (i & 1), e = r * C + j;
            if (warp < 2) {
                const float a = j < r ? c[i] : 0.f;
                if (P) P[e] = a;
                f.A[e] = a * f.b[r];
            } else {
                f.M[e] = j <= r ? c[i] : 0.f;
            }
        }
    }
    __syncthreads();
    // T = (I + A)^-1 by forward substitution, one column per thread, held in registers (the
    // entries above the diagonal are zero, so the sums may start at row 0)
    if (tid < C) {
        const int j = tid;
        float tcol[C];
#pragma unroll
        for (int r = 0; r < C; ++r) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int m = 0; m < r; m += 2) {
                a0 += f.A[r * C + m] * tcol[m];
                if (m + 1 < r) a1 += f.A[r * C + m + 1] * tcol[m + 1];
            }
            tcol[r] = r < j ? 0.f : (r == j ? 1.f : -(a0 + a1));
        }
#pragma unroll
        for (int r = 0; r < C; ++r) f.T[r * C + j] = tcol[r];
    }
    __syncthreads();
    // W = T diag(beta) K_gamma: DK / 8 tiles of 8 channels
    for (int id = warp; id < DK / 8; id += kThreads / 32) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        mma3_tile<C>(c, [&](int m, int kk) { return f.T[m * C + kk] * f.b[kk]; },
                     [&](int kk, int n) { return f.L[kk * LD + 8 * id + n]; }, lane);
        const int g = lane >> 2, t = lane & 3, col = 8 * id + 2 * t;
        f.W[g * LD + col] = c[0];
        f.W[g * LD + col + 1] = c[1];
        f.W[(g + 8) * LD + col] = c[2];
        f.W[(g + 8) * LD + col + 1] = c[3];
    }
    __syncthreads();
    return true;
}

// ---- every chunk's factors into its record: one CTA per (b*h, chunk) ------------------------------
template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kThreads)
chunk_records_kernel(const T* __restrict__ q, const T* __restrict__ k, const void* __restrict__ alpha,
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
    // P = A before beta, straight to the record
    const bool tiles = chunk_products_tiles<DK, C>(f, rec + R::P);
    if (tiles) {
        // Q' = Q_gamma - M W on the warp tiles (8 channels each), straight to the record
        const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
        for (int id = warp; id < DK / 8; id += kThreads / 32) {
            const int col = 8 * id + 2 * t;
            float c[4] = {f.q[g * LD + col], f.q[g * LD + col + 1], f.q[(g + 8) * LD + col],
                          f.q[(g + 8) * LD + col + 1]};
            mma3_tile<C>(c, [&](int m, int kk) { return -f.M[m * C + kk]; },
                         [&](int kk, int n) { return f.W[kk * LD + 8 * id + n]; }, lane);
            *reinterpret_cast<float2*>(rec + R::QP + g * DK + col) = make_float2(c[0], c[1]);
            *reinterpret_cast<float2*>(rec + R::QP + (g + 8) * DK + col) = make_float2(c[2], c[3]);
        }
    }
    for (int e = tid; e < C * DK; e += kThreads) {
        const int r = e / DK, c = e % DK, o = r * LD + c;
        // K_end = sigma_C (g_C / g_r) k';  Q' = Q_gamma - M W (exact form)
        rec[R::W + e] = f.W[o];
        if (tiles) {
            rec[R::KE + e] = f.sg[c] * exp2f(f.LC[c]) * f.k[o];
        } else {
            rec[R::KE + e] = f.sg[c] * exp2f(f.LC[c] - f.L[o]) * f.k[o];
            float qp = exp2f(f.L[o]) * f.q[o];
            for (int j = 0; j <= r; ++j) qp -= f.M[r * C + j] * f.W[j * LD + c];
            rec[R::QP + e] = qp;
        }
    }
    for (int e = tid; e < C * C; e += kThreads) {
        rec[R::T + e] = f.T[e];
        rec[R::M + e] = f.M[e];
    }
    for (int r = tid; r < C; r += kThreads) rec[R::B + r] = f.b[r];
    for (int c = tid; c < DK; c += kThreads) rec[R::GC + c] = f.sg[c] * exp2f(f.LC[c]);
}

// ---- a chunk record in shared memory, for the serial passes ----------------------------------------
// The rows of W, K_end (and Q') are RP = DK + 8 floats apart (the lanes of a warp tile's fragment
// fall on distinct banks), then T, beta and gamma_C as in the record, then (forward pass) M.
template <int DK, int C>
struct Stage {
    static constexpr int RP = DK + 8;
    static constexpr int W = 0, KE = C * RP, T = 2 * C * RP, B = T + C * C, GC = B + C;
    static constexpr int QP = GC + DK, M = QP + C * RP;
    static constexpr int floats_replay = QP, floats_chain = M, floats_fwd = M + C * C;
};
// the record's W, K_end, T, beta, gamma_C, with Q' when with_qp and M when with_m, into a stage
// (one commit group)
template <int DK, int C>
__device__ __forceinline__ void load_stage(float* dst, const float* rec, bool with_qp,
                                           bool with_m = false) {
    using R = Rec<DK, C>;
    using S = Stage<DK, C>;
    constexpr int RC = DK / 4;   // 16-byte pieces per row
    const int nrows = with_qp ? 3 * C : 2 * C;
    for (int i = threadIdx.x; i < nrows * RC; i += kThreads) {
        const int row = i / RC, c4 = 4 * (i % RC), blk = row / C, r = row % C;
        const int src = blk == 0 ? R::W : blk == 1 ? R::KE : R::QP;
        const int d = blk == 0 ? S::W : blk == 1 ? S::KE : S::QP;
        cp16(dst + d + r * S::RP + c4, rec + src + r * DK + c4);
    }
    for (int i = threadIdx.x; i < (C * C + C + DK) / 4; i += kThreads)
        cp16(dst + S::T + 4 * i, rec + R::T + 4 * i);
    if (with_m)
        for (int i = threadIdx.x; i < C * C / 4; i += kThreads) cp16(dst + S::M + 4 * i, rec + R::M + 4 * i);
    cp_commit();
}

}  // namespace

}  // namespace ckda
