// Internal interface between the C-ABI layer (qknr_abi.cu) and the UCPE
// camera-prep launcher (ucpe.cu). Arguments are already validated.
#pragma once

#include "launch.h"

namespace qknr {

struct UcpeArgs {
    const uint8_t* q;  // 16-bit activations [B, N, H, D], dense
    const uint8_t* k;
    const uint8_t* v;
    const float* proj_q;   // [B, N, 4, 4] row-major
    const float* proj_kv;  // [B, N, 4, 4]
    const float* rope_cos; // [N, D/2]
    const float* rope_sin; // [N, D/2]
    uint8_t* q_out;        // 16-bit [B, H, D, N]
    uint8_t* k_out;
    uint8_t* v_out;
    float* inflation_sq;   // [B, H, N] or null (not computed)
    int64_t batch, num_tokens;
    int32_t heads, head_dim;
    int32_t act_f16;  // activations are binary16, else bf16
    float k_scale;
};

// UCPE camera prep (head_dim a multiple of 8 up to 256; pointers 16-byte
// aligned; sizes already checked).
cudaError_t launch_ucpe(const UcpeArgs& a, cudaStream_t stream, LaunchInfo* info);

}  // namespace qknr
