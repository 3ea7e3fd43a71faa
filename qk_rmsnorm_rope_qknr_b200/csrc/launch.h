// Internal interface between the C-ABI layer (qknr_abi.cu) and the kernel
// launchers (rope3d.cu, rope_table.cu). Arguments are already validated.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qknr {

struct Rope3DArgs {
    const uint8_t* qkv;       // bf16 [T, (hq+hk+hv)*D]
    const uint8_t* q_weight;  // bf16 [hq*D] (unused without the norm)
    const uint8_t* k_weight;  // bf16 [hk*D]
    uint8_t* q_out;           // bf16 or E4M3 [T, hq, D]
    uint8_t* k_out;
    uint8_t* v_out;
    int64_t num_tokens;
    int64_t pos_offset;  // reduced modulo ppf*pph*ppw by the host
    int32_t ppf, pph, ppw;
    int32_t cf, ch, cw;
    int32_t hq, hk, hv;
    int32_t is_qk_norm;
    int32_t use_table;      // cos/sin table in shared memory (set by the launcher)
    int32_t table_entries;  // ppf*cf/2 + pph*ch/2 + ppw*cw/2
    float eps;
    float q_scale;
    float v_scale;
    double base;
    // Pipelined (bulk-copy) kernel only:
    int32_t stages;          // ring buffers per token pipeline
    int32_t groups;          // token pipelines per CTA
    int32_t v_bulk;          // bf16 V leaves through a bulk store
    uint32_t stall_tx_bytes; // test hook: extra bytes a stage waits for (0 in use)
    uint64_t wait_limit_ns;  // a wait on a bulk copy gives up after this long
    // Tensor-parallel head slices (see qknr_rope_3d_partial_ssq / _with_ssq):
    int32_t mode;            // 0 whole transform, 1 partial sums only, 2 sums supplied
    float* ssq_out;          // mode 1: [T][2] fp32 (sum Q^2, sum K^2) of this slice
    const float* ssq_in;     // mode 2: [T][2] fp32 sums over all heads of all slices
    int32_t norm_q_elems;    // channels the Q mean runs over (hq*D, or all heads' in mode 2)
    int32_t norm_k_elems;
    int32_t neox_per_axis;   // NeoX halves inside each axis group (groups multiples of 16)
};

enum { kModeWhole = 0, kModePartialSsq = 1, kModeSuppliedSsq = 2 };

struct RopeTableArgs {
    const uint8_t* q;  // 16-bit activations [T, hq, D], token stride q_stride elements
    const uint8_t* k;
    uint8_t* q_out;
    uint8_t* k_out;
    const uint8_t* q_weight;  // [D], the activation type
    const uint8_t* k_weight;
    const uint8_t* table;  // [T, rd] fp32 or the activation type
    int64_t num_tokens;
    int64_t q_stride, k_stride, q_out_stride, k_out_stride;  // elements
    int32_t hq, hk, head_dim, rotary_dim;
    int32_t table_f32;
    int32_t act_f16;  // activations (and a non-fp32 table) are binary16, else bf16
    int32_t interleaved;
    int32_t in_place;  // an output aliases its input
    float eps;
    // Pipelined (bulk-copy) kernel only:
    int32_t stages;           // ring buffers per warp
    uint32_t stall_tx_bytes;  // test hook: extra bytes a buffer waits for (0 in use)
    uint64_t wait_limit_ns;   // a wait on a bulk copy gives up after this long
};

// Launch description returned for the benchmark and tests.
struct LaunchInfo {
    int grid;
    int block;
    int smem;
    int kernel_id;  // which kernel variant ran
};

cudaError_t launch_rope3d(const Rope3DArgs& a, int head_dim, int neox, int fp8,
                          cudaStream_t stream, LaunchInfo* info);

// Status word the pipelined 3D kernel raises (bit 0: a bulk-copy wait timed
// out and the kernel abandoned its remaining tokens). Read on `stream`, after
// the work queued before it; optionally cleared.
cudaError_t read_device_status(uint32_t* out, int clear, cudaStream_t stream);
cudaError_t launch_rope_table(const RopeTableArgs& a, int fast_path, cudaStream_t stream,
                              LaunchInfo* info);

// Status word of the table kernels (bit 0 as for the 3D kernels).
cudaError_t read_table_status(uint32_t* out, int clear, cudaStream_t stream);

}  // namespace qknr
