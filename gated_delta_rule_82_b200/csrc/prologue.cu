// prologue.cu -- q/k prologue: rotary embedding, then the per-head L2 norm.
//
// The rotation pairs (x_i, x_{i+dk/2}) (rotate_half) or (x_{2i}, x_{2i+1}) (interleaved) and
// turns each pair by (pos_offset + t) * theta^(-2i/dk); the L2 norm x / sqrt(sum x^2 + 1e-6)
// follows it ("RoPE into the KDA q/k path" review, sections 2, 3 and 5).
//
// Layout: one CTA handles a run of consecutive tokens (all their heads, q and k).  Each head
// vector is held by a group of GV lanes with 16-byte loads and stores (8 bf16 or 4 fp32 per
// 16 bytes): lane l of the group holds the piece of channels starting at l * EPL and the piece
// starting at dk / 2 + l * EPL, so that the half-split rotation, which pairs channel i with
// i + dk / 2, finds both members of every pair in one lane.  The norm is a GV-lane shuffle
// reduction.  A lane group takes kMaxRounds consecutive head vectors of the run and issues all
// their loads first, so that many bytes are in flight per SM.  Consecutive vectors are
// consecutive heads of one token (when H is a multiple of kMaxRounds, always), so a thread needs
// the sin/cos of its own channels' frequencies at one position: it forms them in registers, again
// only when the token changes.  The kernel reads and writes every q/k element once: it is
// HBM-bound.
#include "fastdiv.h"
#include "internal.cuh"

namespace ckda {

namespace {

constexpr int kPrologueThreads = 256;
constexpr int kMaxRounds = 8;      // head vectors per lane group per batch

// lanes per head vector and lane groups of a CTA (vectors it loads per round)
template <typename T, int DK>
constexpr int vec_lanes() {
    return DK / (2 * ElemsPer16<T>::value);
}
template <typename T, int DK>
constexpr int lane_groups() {
    return kPrologueThreads / vec_lanes<T, DK>();
}

template <typename T, int DK>
__global__ void __launch_bounds__(kPrologueThreads)
qk_prologue_kernel(const T* __restrict__ q, const T* __restrict__ k, T* __restrict__ qo,
                   T* __restrict__ ko, int BT, int T_len, int H, FastDiv hdiv, int tok_per_cta,
                   int l2norm, RopeParams rp, long long pos_offset) {
    constexpr int EPL = ElemsPer16<T>::value;  // elements per 16-byte piece
    constexpr int GV = vec_lanes<T, DK>();     // lanes per head vector
    constexpr int NG = lane_groups<T, DK>();
    constexpr int HALF = DK / 2;
    static_assert(GV >= 1 && GV <= 32, "unsupported head size for this element type");

    __shared__ unsigned long long sfreq[HALF];

    const int tok0 = blockIdx.x * tok_per_cta;
    const int ntok = min(tok_per_cta, BT - tok0);
    const int lg = threadIdx.x / GV, li = threadIdx.x % GV;
    // The run's q vectors are contiguous (tokens x heads x DK), and so are its k vectors: vector
    // v < nvq is q vector v, the others k vector v - nvq; its token in the run is (v mod nvq) / H.
    const int nvq = ntok * H;
    const int nvec = 2 * nvq;
    const int c_lo = li * EPL, c_hi = HALF + li * EPL;     // first channels of the two pieces
    const size_t base = (size_t)tok0 * H * DK;
    // rotation of the first rot channels.  Half-split pairs (i, i + rot / 2) with frequency i:
    // for rot = dk the pieces of one lane pair with each other; for rot = dk / 2 the low piece
    // of lane li < GV / 2 pairs with the low piece of lane li + GV / 2.  Interleaved pairs (2j,
    // 2j + 1) with frequency j lie inside a piece.
    const int rot = rp.rot_dims;
    const bool full = rot == DK;
    const int dl = GV / 2;                                   // partner lanes away (rot = dk / 2)
    const bool rot_lo = rp.enabled && c_lo < rot, rot_hi = rp.enabled && c_hi < rot;
    if (rp.enabled) {
        // frequencies in shared memory (a per-lane index into the kernel-parameter array would
        // serialise in the constant cache)
        for (int i = threadIdx.x; i < HALF; i += blockDim.x) sfreq[i] = rp.turns[i];
        __syncthreads();
    }
    for (int b0 = 0; b0 < nvec; b0 += kMaxRounds * NG) {
        const int v0 = b0 + lg * kMaxRounds;   // this lane group's vectors v0 .. v0 + 7
        // 1. issue every load of this batch
        uint4 raw[kMaxRounds][2];
#pragma unroll
        for (int r = 0; r < kMaxRounds; ++r) {
            const int v = v0 + r;
            if (v < nvec) {
                const bool isk = v >= nvq;
                const T* src = (isk ? k : q) + base + (size_t)(isk ? v - nvq : v) * DK;
                raw[r][0] = __ldcs(reinterpret_cast<const uint4*>(src + c_lo));
                raw[r][1] = __ldcs(reinterpret_cast<const uint4*>(src + c_hi));
            }
        }
        // 2. rotate, normalise, store
        int jc = -1;              // token whose sin/cos are in cs_, sn_
        float cs_[2][EPL], sn_[2][EPL];
#pragma unroll
        for (int r = 0; r < kMaxRounds; ++r) {
            const int v = v0 + r;
            if (b0 + r >= nvec) break;   // CTA-uniform: every vector of this round is past the end
            const bool active = v < nvec;
            const bool isk = v >= nvq;
            const int vi = active ? (isk ? v - nvq : v) : 0;
            float x[2][EPL];
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
                if (active) {
                    if constexpr (EPL == 8) {
                        const uint32_t w[4] = {raw[r][hp].x, raw[r][hp].y, raw[r][hp].z, raw[r][hp].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            x[hp][2 * e] = __uint_as_float(w[e] << 16);
                            x[hp][2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                        }
                    } else {
                        x[hp][0] = __uint_as_float(raw[r][hp].x); x[hp][1] = __uint_as_float(raw[r][hp].y);
                        x[hp][2] = __uint_as_float(raw[r][hp].z); x[hp][3] = __uint_as_float(raw[r][hp].w);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < EPL; ++e) x[hp][e] = 0.f;
                }
            }
            if (rp.enabled) {
                const int j = (int)fastdiv(hdiv, (uint32_t)vi);
                if (j != jc) {
                    jc = j;
                    const long long p = pos_offset + (tok0 + j) % T_len;
#pragma unroll
                    for (int hp = 0; hp < 2; ++hp) {
                        const int c0 = hp ? c_hi : c_lo;
                        // (half-split pairs take the low piece's sin/cos)
                        if (!(hp ? rot_hi && rp.convention == 1 : rot_lo)) continue;
#pragma unroll
                        for (int e = 0; e < EPL; ++e) {
                            // frequency of channel c0 + e: half-split i mod (rot / 2), interleaved i / 2
                            const int fi = rp.convention == 0 ? (c0 + e) % (rot / 2) : (c0 + e) / 2;
                            if (rp.convention == 0 || (e & 1) == 0)
                                rope_sincos(p, sfreq[fi], &sn_[hp][e], &cs_[hp][e]);
                            else {
                                sn_[hp][e] = sn_[hp][e - 1];
                                cs_[hp][e] = cs_[hp][e - 1];
                            }
                        }
                    }
                }
                if (rp.convention == 0 && full) {
                    // pairs (lo e, hi e) of this lane
#pragma unroll
                    for (int e = 0; e < EPL; ++e) {
                        const float a = x[0][e], b = x[1][e];
                        x[0][e] = a * cs_[0][e] - b * sn_[0][e];
                        x[1][e] = b * cs_[0][e] + a * sn_[0][e];
                    }
                } else if (rp.convention == 0) {
                    // rot = dk / 2: low pieces of lanes li and li ^ dl
                    float y[EPL];
#pragma unroll
                    for (int e = 0; e < EPL; ++e) y[e] = __shfl_xor_sync(0xffffffffu, x[0][e], dl);
                    if (rot_lo) {
                        const bool first = li < dl;
#pragma unroll
                        for (int e = 0; e < EPL; ++e)
                            x[0][e] = first ? (x[0][e] * cs_[0][e] - y[e] * sn_[0][e])
                                            : (x[0][e] * cs_[0][e] + y[e] * sn_[0][e]);
                    }
                } else {
#pragma unroll
                    for (int hp = 0; hp < 2; ++hp) {
                        if (!(hp ? rot_hi : rot_lo)) continue;
#pragma unroll
                        for (int e = 0; e < EPL; e += 2) {
                            const float a = x[hp][e], b = x[hp][e + 1];
                            x[hp][e] = a * cs_[hp][e] - b * sn_[hp][e];
                            x[hp][e + 1] = b * cs_[hp][e] + a * sn_[hp][e];
                        }
                    }
                }
            }
            if (l2norm) {
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) ss += x[0][e] * x[0][e] + x[1][e] * x[1][e];
                if constexpr (GV > 1) ss = group_sum<GV>(ss);
                const float rn = rsqrtf(ss + kL2Eps);
#pragma unroll
                for (int e = 0; e < EPL; ++e) {
                    x[0][e] *= rn;
                    x[1][e] *= rn;
                }
            }
            if (active) {
                T* dst = (isk ? ko : qo) + base + (size_t)vi * DK;
                Vec16<T, EPL>::store(dst + c_lo, x[0]);
                Vec16<T, EPL>::store(dst + c_hi, x[1]);
            }
        }
    }
}

template <typename T, int DK>
cudaError_t launch_prologue_t(const void* q, const void* k, void* qo, void* ko, int B, int T_len,
                              int H, int l2norm, const RopeParams& rp, long long pos_offset,
                              cudaStream_t stream) {
    const int BT = B * T_len;
    // tokens per CTA: one batch of kMaxRounds vectors per lane group covers them (at least one
    // token)
    constexpr int per_batch = kMaxRounds * lane_groups<T, DK>();
    const int tpc = max(1, per_batch / (2 * H));
    const int grid = (BT + tpc - 1) / tpc;
    qk_prologue_kernel<T, DK><<<grid, kPrologueThreads, 0, stream>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<T*>(qo),
        static_cast<T*>(ko), BT, T_len, H, make_fastdiv((uint32_t)H), tpc, l2norm, rp,
        pos_offset);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qk_prologue(const void* q, const void* k, void* qo, void* ko, int B, int T_len,
                               int H, int dk, int l2norm, const RopeParams& rp,
                               long long pos_offset, ckda_dtype dtype, cudaStream_t stream) {
#define CKDA_PRO_CASE(TT, D)                                                                  \
    if (dk == D)                                                                             \
        return launch_prologue_t<TT, D>(q, k, qo, ko, B, T_len, H, l2norm, rp, pos_offset, stream);
    if (dtype == CKDA_BF16) {
        CKDA_PRO_CASE(__nv_bfloat16, 16)
        CKDA_PRO_CASE(__nv_bfloat16, 32)
        CKDA_PRO_CASE(__nv_bfloat16, 64)
        CKDA_PRO_CASE(__nv_bfloat16, 128)
    } else {
        CKDA_PRO_CASE(float, 16)
        CKDA_PRO_CASE(float, 32)
        CKDA_PRO_CASE(float, 64)
        CKDA_PRO_CASE(float, 128)
    }
#undef CKDA_PRO_CASE
    return cudaErrorInvalidValue;
}

}  // namespace ckda
