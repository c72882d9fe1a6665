// internal.cuh -- launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include "common.cuh"

namespace ckda {

// Packed sequences of different lengths on one token axis (cu == nullptr: a batch of equal
// lengths).  Sequence s owns tokens cu[s] .. cu[s + 1] - 1; its state rows are s * H + h.
struct PackedSeqs {
    const int* cu;        // device token offsets [n + 1]
    const int* cu_host;   // the same offsets in host memory (sizes the launch)
    int n;                // sequences
};

cudaError_t launch_qk_prologue(const void* q, const void* k, void* qo, void* ko, int B, int T_len,
                               int H, int dk, int l2norm, const RopeParams& rp,
                               long long pos_offset, ckda_dtype dtype, cudaStream_t stream);

// alpha: fp32 gate values, or (gate_logits != 0) logits a of the activation type; with logits
// the kernels form alpha = 2 sigma(a) - 1 and beta = 2 sigma(b) from the fp32 logits in beta.
// G: value heads per q/k head (grouped value heads; 1 = none): q and k have H / G heads and
// value head h reads q/k head h / G.
cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* alpha,
                          const float* beta, float* state, void* out, const long long* pos, int N,
                          int H, int G, int dk, int dv, int l2norm, const RopeParams& rp, float scale,
                          int gate_logits, ckda_dtype dtype, cudaStream_t stream);

// Arguments of the CUDA-core chunked forward.  out and hT are nullable.
struct SimtArgs {
    const void *q, *k, *v, *alpha;
    const float *beta, *h0;
    void* out;
    float* hT;
    int B, T_len;
    const int* cu;   // packed sequences (B = their count), or nullptr
    int H, G, l2norm;
    RopeParams rp;
    float scale;
    long long pos_offset;
    int gate_logits;
};
cudaError_t launch_chunk_simt(const SimtArgs& a, int dk, int dv, int chunk, ckda_dtype dtype,
                              cudaStream_t stream);
cudaError_t launch_chunk_simt(const void* q, const void* k, const void* v, const void* alpha,
                              const float* beta, const float* h0, void* out, float* hT, int B,
                              int T_len, int H, int G, int dk, int dv, int chunk, int l2norm,
                              const RopeParams& rp, float scale, long long pos_offset,
                              int gate_logits, ckda_dtype dtype, const PackedSeqs& pk,
                              cudaStream_t stream);

// Backward of the chunked forward on CUDA cores (fp32 gradients).
struct BwdArgs {
    const void *q, *k, *v, *alpha;
    const float *beta, *h0;
    const void* dout;
    const float* dhT;
    float *dq_out, *dk_out, *dv, *dalpha, *dbeta, *dh0;
    int B, T_len, H, G, l2norm;
    RopeParams rp;
    float scale;
    long long pos_offset;
    int gate_logits;
    ckda_dtype dtype;
};
struct BwdLayout {
    float *records, *states, *dstates, *dq, *dk;
    size_t bytes;
};
BwdLayout bwd_layout(void* ws, int B, int T_len, int H, int dk, int dv);
cudaError_t launch_chunk_bwd(const BwdArgs& a, int dk, int dv, void* workspace,
                             cudaStream_t stream);

// Tensor-core chunked forward (bf16, dk = dv = 128, chunk = 64).
size_t chunk_tc_workspace_bytes(int B, int T_len, int H);
// chunks of packed sequences (sum of ceil(len / 64)) and their workspace
long long packed_chunks(const int* cu_host, int n_seqs);
size_t chunk_tc_workspace_bytes_packed(const int* cu_host, int n_seqs, int H);
// split of the fused tensor-core launch for BH heads of up to NT chunks (n_items chunk-heads in
// all) on nsm SMs: chain CTAs and leading rounds of factor items taken by every CTA
void chunk_tc_plan(int BH, int NT, long long n_items, int nsm, int* n_state, int* lead,
                   double* t_model);
// The segment-parallel pass (batched sequences): workspace, segment count model, launch.
size_t chunk_tc_seg_workspace_bytes(int B, int T_len, int H, int segments);
int chunk_tc_seg_plan(int BH, int NT, int nsm);
cudaError_t launch_chunk_tc_seg(const void* q, const void* k, const void* v, const void* alpha,
                                const float* beta, const float* h0, void* out, float* hT, int B,
                                int T_len, int H, int G, int l2norm, const RopeParams& rp,
                                float scale, long long pos_offset, int gate_logits,
                                void* workspace, int segments, cudaStream_t stream);
cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const void* alpha,
                            const float* beta, const float* h0, void* out, float* hT, int B,
                            int T_len, int H, int G, int l2norm, const RopeParams& rp, float scale,
                            long long pos_offset, int gate_logits, void* workspace, int stages,
                            const PackedSeqs& pk, cudaStream_t stream);

// The forward kernels' device status word on the current device: read once `stream` has
// finished, then cleared (0 = no failure recorded).
cudaError_t device_status_take(cudaStream_t stream, int* code);
// Upper bound of one wait of the fused forward's state role on the current device (0: default).
cudaError_t set_wait_limit_ns(unsigned long long ns);

cudaError_t launch_umma_selftest(const void* A, const void* B, float* D, int M, int N, int K,
                                 int mode, cudaStream_t stream);

}  // namespace ckda
