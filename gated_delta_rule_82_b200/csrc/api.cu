// api.cu -- the C ABI declared in include/ckda.h: argument validation and dispatch.
//
// Everything here runs on the host before any launch.  The library allocates nothing: device
// memory (inputs, outputs, states, workspace) belongs to the caller.
#include <math.h>
#include <string.h>

#include "internal.cuh"
#include "simt_records.h"

using namespace ckda;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_dim(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool supported_chunk(int c) { return c == 16 || c == 32 || c == 64; }

size_t elem_size(ckda_dtype t) { return t == CKDA_BF16 ? 2 : 4; }

// [lo, lo + bytes) intervals intersect?
bool overlap(const void* a, size_t an, const void* b, size_t bn) {
    if (!a || !b || an == 0 || bn == 0) return false;
    uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + bn && y < x + an;
}

ckda_status make_rope(const ckda_flags& f, int dk, RopeParams* rp) {
    memset(rp, 0, sizeof(*rp));
    if (!(f.rope_theta > 0.f)) return CKDA_OK;  // also rejects NaN as "off"
    if (!isfinite(f.rope_theta)) return CKDA_ERR_ARG;
    if (f.rope_convention != 0 && f.rope_convention != 1) return CKDA_ERR_ARG;
    const int rot = f.rope_dims == 0 ? dk : f.rope_dims;
    if (rot != dk && !(rot * 2 == dk && dk >= 32)) return CKDA_ERR_ARG;
    rp->enabled = 1;
    rp->convention = f.rope_convention;
    rp->rot_dims = rot;
    // omega_i = theta^(-2i/rot) ("RoPE review", section 5) as turns per position in 0.64 fixed
    // point, formed in extended precision: 2^64 frac(omega_i / 2 pi)
    const long double two_pi = 6.283185307179586476925286766559005768L;
    for (int i = 0; i < rot / 2; ++i) {
        const long double omega = powl((long double)f.rope_theta, -2.0L * i / rot);
        const long double frac = fmodl(omega / two_pi, 1.0L);
        rp->turns[i] = (unsigned long long)ldexpl(frac, 64);   // exact scaling; truncates
    }
    return CKDA_OK;
}

float resolve_scale(const ckda_flags& f, int dk) {
    return f.scale != 0.f ? f.scale : (float)(1.0 / sqrt((double)dk));
}

bool tc_eligible(int dk, int dv, int chunk, ckda_dtype dtype) {
    return dtype == CKDA_BF16 && dk == 128 && dv == 128 && chunk == 64;
}

// 0 = SIMT, 2 = TC, -1 = unsupported request
int choose_path(int path, int dk, int dv, int chunk, ckda_dtype dtype) {
    if (path == CKDA_PATH_SIMT) return CKDA_PATH_SIMT;
    if (path == CKDA_PATH_TC) return tc_eligible(dk, dv, chunk, dtype) ? CKDA_PATH_TC : -1;
    if (path == CKDA_PATH_AUTO) return tc_eligible(dk, dv, chunk, dtype) ? CKDA_PATH_TC : CKDA_PATH_SIMT;
    return -1;
}

ckda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA; }

}  // namespace

extern "C" {

int ckda_abi_version(void) { return CKDA_ABI_VERSION; }

const char* ckda_strerror(ckda_status s) {
    switch (s) {
        case CKDA_OK: return "success";
        case CKDA_ERR_NULL: return "a required pointer is NULL";
        case CKDA_ERR_SHAPE: return "a size is out of range";
        case CKDA_ERR_UNSUPPORTED: return "head size, chunk, dtype or path not supported";
        case CKDA_ERR_ALIGN: return "an array pointer is not 16-byte aligned";
        case CKDA_ERR_WORKSPACE: return "workspace missing or too small";
        case CKDA_ERR_CUDA: return "a CUDA runtime call failed";
        case CKDA_ERR_ARG: return "invalid argument";
        case CKDA_ERR_DEVICE_STATUS: return "a kernel recorded a failure on the device";
    }
    return "unknown status";
}

ckda_status ckda_last_device_status(ckda_stream_t stream, int* code) {
    int v = 0;
    if (device_status_take((cudaStream_t)stream, &v) != cudaSuccess) return CKDA_ERR_CUDA;
    if (code) *code = v;
    return v == 0 ? CKDA_OK : CKDA_ERR_DEVICE_STATUS;
}

ckda_status ckda_set_wait_limit_ns(unsigned long long ns) {
    return from_cuda(set_wait_limit_ns(ns));
}

ckda_status ckda_qk_prologue(const void* q, const void* k, void* q_out, void* k_out, int B, int T,
                             int H, int dk, ckda_flags flags, ckda_dtype dtype,
                             long long pos_offset, ckda_stream_t stream) {
    if (!q || !k || !q_out || !k_out) return CKDA_ERR_NULL;
    if (dtype != CKDA_F32 && dtype != CKDA_BF16) return CKDA_ERR_UNSUPPORTED;
    if (B < 1 || T < 1 || H < 1) return CKDA_ERR_SHAPE;
    if ((long long)B * T * H * dk > (1ll << 40)) return CKDA_ERR_SHAPE;
    if (!supported_dim(dk)) return CKDA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out)) return CKDA_ERR_ALIGN;
    size_t bytes = (size_t)B * T * H * dk * elem_size(dtype);
    // in-place is allowed; partial overlaps and q_out aliasing k are not
    if ((q_out != q && overlap(q_out, bytes, q, bytes)) || overlap(q_out, bytes, k, bytes) ||
        (k_out != k && overlap(k_out, bytes, k, bytes)) || overlap(k_out, bytes, q, bytes) ||
        overlap(q_out, bytes, k_out, bytes))
        return CKDA_ERR_ARG;
    RopeParams rp;
    ckda_status st = make_rope(flags, dk, &rp);
    if (st != CKDA_OK) return st;
    return from_cuda(launch_qk_prologue(q, k, q_out, k_out, B, T, H, dk, flags.l2norm ? 1 : 0, rp,
                                        pos_offset, dtype, (cudaStream_t)stream));
}

size_t ckda_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, ckda_dtype dtype,
                                int path) {
    if (B < 1 || T < 1 || H < 1) return (size_t)-1;
    if (!supported_dim(dk) || !supported_dim(dv) || !supported_chunk(chunk)) return (size_t)-1;
    if (dtype != CKDA_F32 && dtype != CKDA_BF16) return (size_t)-1;
    int p = choose_path(path, dk, dv, chunk, dtype);
    if (p < 0) return (size_t)-1;
    if (p == CKDA_PATH_TC) return chunk_tc_workspace_bytes(B, T, H);
    return 0;
}

}  // extern "C"

namespace {

// Offsets of packed sequences, checked on the host: cu[0] = 0, non-decreasing.  Returns the
// token count cu[n], or -1.
long long packed_tokens(const int* cu_host, int n) {
    if (!cu_host || n < 1 || cu_host[0] != 0) return -1;
    for (int s = 0; s < n; ++s)
        if (cu_host[s + 1] < cu_host[s]) return -1;
    return cu_host[n];
}

// The forward over a batch (pk.cu == nullptr: B rows of T tokens) or over packed sequences
// (pk.n sequences on one axis of T tokens; states per sequence).
ckda_status fwd_impl(const void* q, const void* k, const void* v, const void* alpha,
                     const float* beta, const float* h0, void* out, float* hT, int B, int T, int H,
                     int dk, int dv, int chunk, ckda_flags flags, ckda_dtype dtype,
                     long long pos_offset, void* workspace, size_t workspace_bytes,
                     const PackedSeqs& pk, cudaStream_t stream, int segments = 1) {
    const bool packed = pk.cu != nullptr;
    if (!q || !k || !v || !alpha || !beta || !out) return CKDA_ERR_NULL;
    if (dtype != CKDA_F32 && dtype != CKDA_BF16) return CKDA_ERR_UNSUPPORTED;
    if (B < 1 || T < (packed ? 0 : 1) || H < 1) return CKDA_ERR_SHAPE;
    const long long ntok = packed ? (long long)T : (long long)B * T;   // tokens on the token axis
    const long long nrows = packed ? (long long)pk.n : (long long)B;    // initial / final states
    if (ntok * H * 128 > (1ll << 40) || nrows * H * 128 * 128 > (1ll << 40)) return CKDA_ERR_SHAPE;
    const long long chunks16 = packed ? ntok / 16 + nrows : (long long)B * ((T + 15) / 16);
    if (chunks16 * H > 0x7fffffffll) return CKDA_ERR_SHAPE;
    if (!supported_dim(dk) || !supported_dim(dv) || !supported_chunk(chunk)) return CKDA_ERR_UNSUPPORTED;
    int p = choose_path(flags.path, dk, dv, chunk, dtype);
    if (p < 0) return flags.path == CKDA_PATH_TC ? CKDA_ERR_UNSUPPORTED : CKDA_ERR_ARG;
    const void* ptrs[] = {q, k, v, alpha, beta, h0, out, hT};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return CKDA_ERR_ALIGN;
    if (flags.qk_heads < 0 || (flags.qk_heads > 0 && H % flags.qk_heads != 0)) return CKDA_ERR_ARG;
    const int G = flags.qk_heads > 0 ? H / flags.qk_heads : 1;   // value heads per q/k head
    const size_t es = elem_size(dtype);
    const size_t nqk = (size_t)ntok * (H / G) * dk, nv = (size_t)ntok * H * dv;
    const size_t nalpha = (size_t)ntok * H * dk;
    const size_t nst = (size_t)nrows * H * dk * dv;
    // outputs must not overlap any input (hT == h0 exactly is allowed: each state is read
    // completely before it is written)
    if (flags.gate_logits != 0 && flags.gate_logits != 1) return CKDA_ERR_ARG;
    const size_t asz = nalpha * (flags.gate_logits ? es : 4);   // gate values fp32, logits `dtype`
    const void* ins[] = {q, k, v, alpha, beta};
    const size_t insz[] = {nqk * es, nqk * es, nv * es, asz, (size_t)ntok * H * 4};
    for (int i = 0; i < 5; ++i) {
        if (overlap(out, nv * es, ins[i], insz[i])) return CKDA_ERR_ARG;
        if (hT && overlap(hT, nst * 4, ins[i], insz[i])) return CKDA_ERR_ARG;
    }
    if (hT && overlap(hT, nst * 4, out, nv * es)) return CKDA_ERR_ARG;
    if (h0 && overlap(h0, nst * 4, out, nv * es)) return CKDA_ERR_ARG;
    if (h0 && hT && hT != h0 && overlap(hT, nst * 4, h0, nst * 4)) return CKDA_ERR_ARG;
    if (flags.stages < 0 || flags.stages > 3) return CKDA_ERR_ARG;
    RopeParams rp;
    ckda_status st = make_rope(flags, dk, &rp);
    if (st != CKDA_OK) return st;
    const float scale = resolve_scale(flags, dk);
    const int l2 = flags.l2norm ? 1 : 0;
    if (segments != 1 && (p != CKDA_PATH_TC || packed)) return CKDA_ERR_UNSUPPORTED;
    if (p == CKDA_PATH_TC) {
        size_t need = packed          ? chunk_tc_workspace_bytes_packed(pk.cu_host, pk.n, H)
                      : segments != 1 ? chunk_tc_seg_workspace_bytes(B, T, H, segments)
                                      : chunk_tc_workspace_bytes(B, T, H);
        if (need > 0 && (!workspace || workspace_bytes < need)) return CKDA_ERR_WORKSPACE;
        if (workspace && !aligned16(workspace)) return CKDA_ERR_ALIGN;
        const void* all[] = {q, k, v, alpha, beta, h0, out, hT};
        const size_t allsz[] = {nqk * es, nqk * es, nv * es, asz, (size_t)ntok * H * 4,
                                nst * 4, nv * es, nst * 4};
        for (int i = 0; i < 8; ++i)
            if (all[i] && overlap(workspace, need, all[i], allsz[i])) return CKDA_ERR_ARG;
        if (segments != 1)
            return from_cuda(launch_chunk_tc_seg(q, k, v, alpha, beta, h0, out, hT, B, T, H, G, l2,
                                                 rp, scale, pos_offset, flags.gate_logits,
                                                 workspace, segments, stream));
        return from_cuda(launch_chunk_tc(q, k, v, alpha, beta, h0, out, hT, B, T, H, G, l2, rp,
                                         scale, pos_offset, flags.gate_logits, workspace,
                                         flags.stages, pk, stream));
    }
    // CUDA-core path: the record form when the caller gives it a workspace (batched sequences)
    if (!packed && workspace) {
        const size_t need = simt_records_bytes(B, T, H, dk);
        if (workspace_bytes >= need) {
            if (!aligned16(workspace)) return CKDA_ERR_ALIGN;
            const void* all[] = {q, k, v, alpha, beta, h0, out, hT};
            const size_t allsz[] = {nqk * es, nqk * es, nv * es, asz, (size_t)ntok * H * 4,
                                    nst * 4, nv * es, nst * 4};
            for (int i = 0; i < 8; ++i)
                if (all[i] && overlap(workspace, need, all[i], allsz[i])) return CKDA_ERR_ARG;
            const SimtArgs a{q, k, v, alpha, beta, h0, out, hT, B, T, nullptr, H, G, l2, rp,
                             scale, pos_offset, flags.gate_logits};
            return from_cuda(launch_chunk_simt_records(a, dk, dv, dtype, workspace, stream));
        }
    }
    return from_cuda(launch_chunk_simt(q, k, v, alpha, beta, h0, out, hT, B, T, H, G, dk, dv, chunk,
                                       l2, rp, scale, pos_offset, flags.gate_logits, dtype, pk,
                                       stream));
}

}  // namespace

extern "C" {

ckda_status ckda_fwd_chunked(const void* q, const void* k, const void* v, const void* alpha,
                             const float* beta, const float* h0, void* out, float* hT, int B,
                             int T, int H, int dk, int dv, int chunk, ckda_flags flags,
                             ckda_dtype dtype, long long pos_offset, void* workspace,
                             size_t workspace_bytes, ckda_stream_t stream) {
    const PackedSeqs none{nullptr, nullptr, 0};
    return fwd_impl(q, k, v, alpha, beta, h0, out, hT, B, T, H, dk, dv, chunk, flags, dtype,
                    pos_offset, workspace, workspace_bytes, none, (cudaStream_t)stream);
}

size_t ckda_fwd_simt_workspace_bytes(int B, int T, int H, int dk, int dv) {
    if (B < 1 || T < 1 || H < 1) return (size_t)-1;
    if (!supported_dim(dk) || !supported_dim(dv)) return (size_t)-1;
    if ((long long)B * T * H * 128 > (1ll << 40)) return (size_t)-1;
    return simt_records_bytes(B, T, H, dk);
}

int ckda_fwd_segments_auto(int B, int T, int H) {
    if (B < 1 || T < 1 || H < 1 || (long long)B * H > 0x7fffffffll) return 1;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    return chunk_tc_seg_plan(B * H, (T + 63) / 64, nsm);
}

size_t ckda_fwd_segmented_workspace_bytes(int B, int T, int H, int dk, int dv, int segments) {
    if (B < 1 || T < 1 || H < 1 || segments < 1) return (size_t)-1;
    if (dk != 128 || dv != 128) return (size_t)-1;
    if ((long long)B * T * H * 128 > (1ll << 40)) return (size_t)-1;
    return chunk_tc_seg_workspace_bytes(B, T, H, segments);
}

ckda_status ckda_fwd_segmented(const void* q, const void* k, const void* v, const void* alpha,
                               const float* beta, const float* h0, void* out, float* hT, int B,
                               int T, int H, int dk, int dv, ckda_flags flags, ckda_dtype dtype,
                               long long pos_offset, int segments, void* workspace,
                               size_t workspace_bytes, ckda_stream_t stream) {
    if (segments < 1) return CKDA_ERR_ARG;
    if (flags.path == CKDA_PATH_SIMT) return CKDA_ERR_UNSUPPORTED;
    flags.stages = 0;   // (ignored here: segments = 1 is the single fused launch)
    const PackedSeqs none{nullptr, nullptr, 0};
    return fwd_impl(q, k, v, alpha, beta, h0, out, hT, B, T, H, dk, dv, 64, flags, dtype,
                    pos_offset, workspace, workspace_bytes, none, (cudaStream_t)stream, segments);
}

size_t ckda_fwd_varlen_workspace_bytes(const int* cu_seqlens_host, int n_seqs, int H, int dk,
                                       int dv, int chunk, ckda_dtype dtype, int path) {
    if (packed_tokens(cu_seqlens_host, n_seqs) < 0 || H < 1) return (size_t)-1;
    if (!supported_dim(dk) || !supported_dim(dv) || !supported_chunk(chunk)) return (size_t)-1;
    if (dtype != CKDA_F32 && dtype != CKDA_BF16) return (size_t)-1;
    int p = choose_path(path, dk, dv, chunk, dtype);
    if (p < 0) return (size_t)-1;
    if (p == CKDA_PATH_TC) return chunk_tc_workspace_bytes_packed(cu_seqlens_host, n_seqs, H);
    return 0;
}

ckda_status ckda_fwd_varlen(const void* q, const void* k, const void* v, const void* alpha,
                            const float* beta, const float* h0, void* out, float* hT,
                            const int* cu_seqlens, const int* cu_seqlens_host, int n_seqs, int H,
                            int dk, int dv, int chunk, ckda_flags flags, ckda_dtype dtype,
                            long long pos_offset, void* workspace, size_t workspace_bytes,
                            ckda_stream_t stream) {
    if (!cu_seqlens || !cu_seqlens_host) return CKDA_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) return CKDA_ERR_ALIGN;
    if (n_seqs < 1) return CKDA_ERR_SHAPE;
    const long long T = packed_tokens(cu_seqlens_host, n_seqs);
    if (T < 0) return CKDA_ERR_ARG;
    if (T > 0x7fffffffll) return CKDA_ERR_SHAPE;
    const PackedSeqs pk{cu_seqlens, cu_seqlens_host, n_seqs};
    return fwd_impl(q, k, v, alpha, beta, h0, out, hT, 1, (int)T, H, dk, dv, chunk, flags, dtype,
                    pos_offset, workspace, workspace_bytes, pk, (cudaStream_t)stream);
}

ckda_status ckda_decode_step(const void* q, const void* k, const void* v, const void* alpha,
                             const float* beta, float* state, void* out, const long long* pos,
                             int N, int H, int dk, int dv, ckda_flags flags, ckda_dtype dtype,
                             ckda_stream_t stream) {
    if (!q || !k || !v || !alpha || !beta || !state || !out) return CKDA_ERR_NULL;
    if (dtype != CKDA_F32 && dtype != CKDA_BF16) return CKDA_ERR_UNSUPPORTED;
    if (N < 1 || H < 1) return CKDA_ERR_SHAPE;
    if ((long long)N * H * dk * dv > (1ll << 40)) return CKDA_ERR_SHAPE;
    if (!supported_dim(dk) || !supported_dim(dv)) return CKDA_ERR_UNSUPPORTED;
    RopeParams rp;
    ckda_status st = make_rope(flags, dk, &rp);
    if (st != CKDA_OK) return st;
    if (rp.enabled && !pos) return CKDA_ERR_NULL;
    const void* ptrs[] = {q, k, v, alpha, beta, state, out};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return CKDA_ERR_ALIGN;
    if (rp.enabled && (reinterpret_cast<uintptr_t>(pos) & 7u)) return CKDA_ERR_ALIGN;
    if (flags.qk_heads < 0 || (flags.qk_heads > 0 && H % flags.qk_heads != 0)) return CKDA_ERR_ARG;
    const int G = flags.qk_heads > 0 ? H / flags.qk_heads : 1;   // value heads per q/k head
    const size_t es = elem_size(dtype);
    const size_t nst = (size_t)N * H * dk * dv * 4;
    if (flags.gate_logits != 0 && flags.gate_logits != 1) return CKDA_ERR_ARG;
    const void* ins[] = {q, k, v, alpha, beta};
    const size_t insz[] = {(size_t)N * (H / G) * dk * es, (size_t)N * (H / G) * dk * es,
                           (size_t)N * H * dv * es, (size_t)N * H * dk * (flags.gate_logits ? es : 4),
                           (size_t)N * H * 4};
    for (int i = 0; i < 5; ++i) {
        if (overlap(out, (size_t)N * H * dv * es, ins[i], insz[i])) return CKDA_ERR_ARG;
        if (overlap(state, nst, ins[i], insz[i])) return CKDA_ERR_ARG;
    }
    if (overlap(state, nst, out, (size_t)N * H * dv * es)) return CKDA_ERR_ARG;
    return from_cuda(launch_decode(q, k, v, alpha, beta, state, out, rp.enabled ? pos : nullptr,
                                   N, H, G, dk, dv, flags.l2norm ? 1 : 0, rp,
                                   resolve_scale(flags, dk), flags.gate_logits, dtype,
                                   (cudaStream_t)stream));
}

size_t ckda_bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
    if (B < 1 || T < 1 || H < 1) return (size_t)-1;
    if (!supported_dim(dk) || !supported_dim(dv)) return (size_t)-1;
    if ((long long)B * T * H * 128 > (1ll << 40)) return (size_t)-1;
    return bwd_layout(nullptr, B, T, H, dk, dv).bytes;
}

ckda_status ckda_bwd_chunked(const void* q, const void* k, const void* v, const void* alpha,
                             const float* beta, const float* h0, const void* dout,
                             const float* dhT, float* dq, float* dk, float* dv, float* dalpha,
                             float* dbeta, float* dh0, int B, int T, int H, int dk_, int dv_,
                             ckda_flags flags, ckda_dtype dtype, long long pos_offset,
                             void* workspace, size_t workspace_bytes, ckda_stream_t stream) {
    if (!q || !k || !v || !alpha || !beta || !dout || !dq || !dk || !dv || !dalpha || !dbeta)
        return CKDA_ERR_NULL;
    if (dtype != CKDA_F32 && dtype != CKDA_BF16) return CKDA_ERR_UNSUPPORTED;
    if (B < 1 || T < 1 || H < 1) return CKDA_ERR_SHAPE;
    if ((long long)B * T * H * 128 > (1ll << 40) || (long long)B * H * 128 * 128 > (1ll << 40))
        return CKDA_ERR_SHAPE;
    if ((long long)B * H * ((T + 15) / 16) > 0x7fffffffll) return CKDA_ERR_SHAPE;
    if (!supported_dim(dk_) || !supported_dim(dv_)) return CKDA_ERR_UNSUPPORTED;
    if (flags.qk_heads < 0 || (flags.qk_heads > 0 && H % flags.qk_heads != 0)) return CKDA_ERR_ARG;
    if (flags.gate_logits != 0 && flags.gate_logits != 1) return CKDA_ERR_ARG;
    const void* ptrs[] = {q, k, v, alpha, beta, h0, dout, dhT, dq, dk, dv, dalpha, dbeta, dh0,
                          workspace};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return CKDA_ERR_ALIGN;
    const size_t need = ckda_bwd_workspace_bytes(B, T, H, dk_, dv_);
    if (!workspace || workspace_bytes < need) return CKDA_ERR_WORKSPACE;
    const int G = flags.qk_heads > 0 ? H / flags.qk_heads : 1;
    const size_t es = elem_size(dtype), ntok = (size_t)B * T;
    const size_t nqk = ntok * (H / G) * dk_, nv = ntok * H * dv_, nal = ntok * H * dk_;
    const size_t nst = (size_t)B * H * dk_ * dv_;
    // outputs (fp32) against every input and each other; the workspace against all of them
    const void* ins[] = {q, k, v, alpha, beta, h0, dout, dhT};
    const size_t insz[] = {nqk * es, nqk * es, nv * es, nal * (flags.gate_logits ? es : 4),
                           ntok * H * 4, nst * 4, nv * es, nst * 4};
    void* outs[] = {dq, dk, dv, dalpha, dbeta, dh0, workspace};
    const size_t outsz[] = {nqk * 4, nqk * 4, nv * 4, nal * 4, ntok * H * 4, nst * 4, need};
    for (int i = 0; i < 7; ++i) {
        for (int j = 0; j < 8; ++j)
            if (outs[i] && overlap(outs[i], outsz[i], ins[j], insz[j])) return CKDA_ERR_ARG;
        for (int j = 0; j < i; ++j)
            if (outs[i] && outs[j] && overlap(outs[i], outsz[i], outs[j], outsz[j])) return CKDA_ERR_ARG;
    }
    BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.h0 = h0; a.dout = dout;
    a.dhT = dhT; a.dq_out = dq; a.dk_out = dk; a.dv = dv; a.dalpha = dalpha; a.dbeta = dbeta;
    a.dh0 = dh0; a.B = B; a.T_len = T; a.H = H; a.G = G; a.l2norm = flags.l2norm ? 1 : 0;
    ckda_status st = make_rope(flags, dk_, &a.rp);
    if (st != CKDA_OK) return st;
    a.scale = resolve_scale(flags, dk_);
    a.pos_offset = pos_offset;
    a.gate_logits = flags.gate_logits;
    a.dtype = dtype;
    return from_cuda(launch_chunk_bwd(a, dk_, dv_, workspace, (cudaStream_t)stream));
}

ckda_status ckda_selftest_umma(const void* A, const void* B, float* D, int M, int N, int K,
                               int b_mn_major, ckda_stream_t stream) {
    if (!A || !B || !D) return CKDA_ERR_NULL;
    if (M != 64 && M != 128) return CKDA_ERR_UNSUPPORTED;
    if (N < 16 || N > 256 || N % 16) return CKDA_ERR_UNSUPPORTED;
    if (K < 64 || K > 256 || K % 64) return CKDA_ERR_UNSUPPORTED;
    if ((b_mn_major & ~7) || (b_mn_major & 6) == 6) return CKDA_ERR_ARG;
    if ((b_mn_major & 1) && N % 64 && N != 32) return CKDA_ERR_UNSUPPORTED;
    if ((b_mn_major & 6) && M != 128) return CKDA_ERR_UNSUPPORTED;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D)) return CKDA_ERR_ALIGN;
    return from_cuda(launch_umma_selftest(A, B, D, M, N, K, b_mn_major,
                                          (cudaStream_t)stream));
}

}  // extern "C"
