// mk_kernels.h -- launch entry points of the device code (internal).
#pragma once
#include <cuda_runtime.h>

#include "mk_internal.h"

namespace mk {

// Step parameters in device memory for the multi-kernel baseline, so that the
// per-op launches can be replayed from a CUDA graph.
struct StepBuf {
    int token;
    int pos;
    int pad[2];
};

struct BaselineShape {
    int n_sm;
    int lm_blocks;  // blocks of the LM-head launch (= partial argmax slots)
};

size_t megakernel_smem_bytes(int ring_stages, int stage_bytes);
cudaError_t prepare_megakernel(int ring_stages, int stage_bytes, int* max_blocks_per_sm);
// Kernel instantiation for a schedule: 1 or 2 when every GEMV-type instruction
// has that many 8-column chunks per consumer thread (fused FFN, no optional L2
// prefetch), else 0 (the general kernel).
int megakernel_variant(const DevParams& p, bool fused_ffn);
// Bytes between the weight rows of a ring stage beyond the row, for instantiation `variant`.
int megakernel_row_pad(int variant);
cudaError_t launch_megakernel(const DevParams& p, const StepArgs& a, int n_sm, int variant, cudaStream_t stream);

// dst[c][r] = src[r][c] for a row-major bf16 matrix of rows x cols (one-time,
// at set-up: the fused FFN streams the down-projection by its input index).
cudaError_t launch_transpose_bf16(const uint16_t* src, uint16_t* dst, int rows, int cols, cudaStream_t stream);

int baseline_lm_blocks(const DevParams& p, int n_sm);
cudaError_t prepare_baseline();
cudaError_t launch_baseline_set_step(const DevParams& p, StepBuf* sb, int token, int pos, cudaStream_t stream);
cudaError_t launch_baseline_layers(const DevParams& p, const uint16_t* const* wt_host, const StepBuf* sb,
                                   const BaselineShape& bs, float* logits, cudaStream_t stream);

}  // namespace mk
