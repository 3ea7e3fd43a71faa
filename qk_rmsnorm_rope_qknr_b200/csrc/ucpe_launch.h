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

// What only the warp-specialised kernel needs (kept out of UcpeArgs, whose
// layout the other two kernels' register allocation is sensitive to).
struct UcpeControl {
    int32_t device_inputs;    // q, k, v are device memory (the kernel reads them by tensor maps)
    uint32_t stall_tx_bytes;  // test hook: extra bytes a ring stage waits for (0 in use)
    uint64_t wait_limit_ns;   // a wait on a copy or on another warp gives up after this long
};

// UCPE camera prep (head_dim a multiple of 8 up to 256; pointers 16-byte
// aligned; sizes already checked).
cudaError_t launch_ucpe(const UcpeArgs& a, const UcpeControl& ctl, cudaStream_t stream,
                        LaunchInfo* info);

// Status word of the camera-prep kernels (bit 0: a wait ran past its limit and
// the launch abandoned its remaining steps), read on `stream`; optionally
// cleared.
cudaError_t read_ucpe_status(uint32_t* out, int clear, cudaStream_t stream);

}  // namespace qknr
