// simt_records.h -- the record form of the CUDA-core chunked forward (chunk_simt.cu): its
// workspace and its launch.
#pragma once

#include <cstddef>

#include "internal.cuh"

namespace ckda {

// Bytes of the factor records of every chunk of 16 tokens, [B*H][ceil(T/16)][3*16*dk + 3*16*16 +
// 16 + dk] fp32 (batched sequences).
size_t simt_records_bytes(int B, int T_len, int H, int dk);
// The records of every chunk (chunk-parallel), then the pass over them: one CTA per (batch*head,
// 16 state columns).  `workspace` holds simt_records_bytes(...) and is 16-byte aligned.
cudaError_t launch_chunk_simt_records(const SimtArgs& a, int dk, int dv, ckda_dtype dtype,
                                      void* workspace, cudaStream_t stream);

}  // namespace ckda
