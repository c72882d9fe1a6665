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

// ---- warp-level tensor-core tiles with fp32-grade products ------------------------------------
// mma.sync m16n8k8 with tf32 operands, each operand split into a tf32 head and a tf32 tail
// (x = hi + lo, lo the rounded remainder): a b = a_hi b_hi + a_hi b_lo + a_lo b_hi up to a relative
// 2^-21, i.e. the product of two fp32 values to about fp32 precision ("3xTF32").  Fragment layout
// (PTX ISA, mma.m16n8k8 .tf32), g = lane / 4, t = lane % 4: A a0 = A[g][t], a1 = A[g+8][t],
// a2 = A[g][t+4], a3 = A[g+8][t+4]; B b0 = B[t][g], b1 = B[t+4][g]; D d0 = D[g][2t],
// d1 = D[g][2t+1], d2 = D[g+8][2t], d3 = D[g+8][2t+1].
__device__ __forceinline__ uint32_t f2tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = f2tf32(x);
    lo = f2tf32(x - __uint_as_float(hi));
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
