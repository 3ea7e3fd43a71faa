/*
 * qknr.h -- C ABI of libqknr.so: fused Q/K RMSNorm + rotary position embedding
 * (with V copy and optional FP8 E4M3 output) for B200 (sm_100a).
 *
 * Two entry points, one per contract that the source pages state:
 *
 *   qknr_rope_table  -- "vllm_omni.diffusion.layers.fused_qk_norm_rope"
 *                       (vLLM-Omni API docs): module description (public
 *                       contract bullets) and fused_qk_norm_rope(...).
 *   qknr_rope_3d     -- "flashinfer.norm.fused_qk_rmsnorm_rope" (FlashInfer
 *                       API docs): summary, Parameters, Returns.
 *
 * and the camera-branch transform that runs beside them in the same block:
 *
 *   qknr_ucpe_cam_prep -- "vllm_omni.diffusion.models.sana_wm.ucpe"
 *                       (vLLM-Omni API docs): cam_prep_func, its
 *                       description, Parameters and Returns.
 *
 * Common rules
 *   - Pointers are plain addresses that the current CUDA device can read or
 *     write: device memory of that device, managed memory, or page-locked host
 *     memory registered with CUDA (then the kernel reads and writes it across
 *     the bus). Anything else is rejected with QKNR_ERR_POINTER before any
 *     launch.
 *   - The caller owns every buffer (destination-passing); the library never
 *     allocates, frees or synchronises. Work is queued on `cuda_stream`
 *     (a cudaStream_t; NULL = the legacy default stream) and the call returns
 *     at once. A fault inside the kernel surfaces at the caller's next
 *     synchronisation on that stream.
 *   - Every entry point returns a qknr_status. Nothing is thrown across the
 *     ABI and nothing is written when the status is not QKNR_OK.
 *     qknr_last_error_detail() names the argument that failed, for this thread.
 *   - num_tokens == 0 is a valid no-op (QKNR_OK, no launch).
 *   - bf16 is bfloat16 (the upper half of an IEEE binary32), f16 is IEEE
 *     binary16, E4M3 is the OCP FP8 E4M3FN format (bias 7, largest finite
 *     448, no infinities); conversions to bf16 and f16 round to nearest even,
 *     conversions to E4M3 round to nearest even and saturate to +-448.
 *   - All arithmetic is fp32; each output element is rounded once.
 *
 * Thread safety: calls may come from several host threads and streams at once.
 */
#ifndef QKNR_H_
#define QKNR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QKNR_ABI_VERSION 4

typedef enum {
    QKNR_OK = 0,
    QKNR_ERR_NULL = 1,        /* a pointer that the call needs is NULL               */
    QKNR_ERR_SHAPE = 2,       /* sizes or parameters break the contract              */
    QKNR_ERR_UNSUPPORTED = 3, /* allowed by the pages but not built (YARN, factor!=1) */
    QKNR_ERR_ALIGN = 4,       /* a pointer or row stride misses the 16-byte rule     */
    QKNR_ERR_ALIAS = 5,       /* an output overlaps an input it may not overlap      */
    QKNR_ERR_POINTER = 6,     /* a pointer the current device cannot access          */
    QKNR_ERR_CUDA = 7         /* the CUDA runtime refused the launch                 */
} qknr_status;

typedef enum {
    QKNR_DT_BF16 = 0,
    QKNR_DT_F32 = 1,
    QKNR_DT_E4M3 = 2,
    QKNR_DT_F16 = 3 /* IEEE binary16 */
} qknr_dtype;

/*
 * Table-driven per-head Q/K RMSNorm + RoPE
 * ("vllm_omni.diffusion.layers.fused_qk_norm_rope": contract bullets and
 * fused_qk_norm_rope).
 *
 * For every token t and every head h of q (and of k, with k's weight):
 *   y[d]   = x[d] / sqrt(mean_d'(x[d']^2) + eps) * weight[d]      (d < head_dim)
 *   pair j = (2j, 2j+1) if interleaved, else (j, j + rotary_dim/2)  (j < rotary_dim/2)
 *   c = rope_table[t][j], s = rope_table[t][rotary_dim/2 + j]
 *   out[a] = y[a] c - y[b] s,  out[b] = y[b] c + y[a] s;  channels >= rotary_dim: out = y
 *
 * act_dtype     QKNR_DT_BF16 or QKNR_DT_F16: the type of q, k, their outputs
 *               and the weights (the "activation dtype").
 * q, k          [num_tokens, heads, head_dim] of act_dtype: heads dense inside
 *               a token, tokens q_token_stride / k_token_stride ELEMENTS apart
 *               (0 = dense, heads*head_dim). Read only.
 * q_out, k_out  act_dtype, same shape, their own token strides (0 = dense). May
 *               equal q / k exactly (in place, then with the same stride);
 *               any other overlap with an input is QKNR_ERR_ALIAS.
 * q_weight, k_weight  act_dtype [head_dim].
 * rope_table    [num_tokens, rotary_dim], dense, QKNR_DT_F32 or act_dtype (the
 *               contract bullets allow exactly these two table types):
 *               columns [0, rotary_dim/2) hold cos(theta_j), the rest sin(theta_j).
 *               Any other act_dtype, or a 16-bit table of the other 16-bit
 *               type, is QKNR_ERR_SHAPE.
 * head_dim      1..256; rotary_dim 0 means head_dim, else even and <= head_dim.
 * heads_q, heads_k >= 0 (a tensor with 0 heads is neither read nor written and
 *               its pointers may be NULL).
 * eps           >= 0.
 * Range: sums of squares are accumulated in fp32, so a head whose sum of
 * squares overflows fp32 (|x| above about 1e18 at head_dim 128) comes out as
 * zeros or NaN; with eps == 0 an all-zero head comes out as NaN (0/0), as in
 * the definition.
 * Fast path: every pointer and token stride 16-byte aligned, head_dim a
 * multiple of 16 and rotary_dim a multiple of 16 (half-split) or 8
 * (interleaved). Other valid inputs run a general kernel (2-byte alignment).
 */
int qknr_rope_table(const void* q, const void* k, void* q_out, void* k_out,
                    const void* q_weight, const void* k_weight, const void* rope_table,
                    int32_t table_dtype, int32_t act_dtype, int64_t num_tokens, int32_t heads_q,
                    int32_t heads_k,
                    int32_t head_dim, int32_t rotary_dim, int64_t q_token_stride,
                    int64_t k_token_stride, int64_t q_out_token_stride,
                    int64_t k_out_token_stride, float eps, int32_t interleaved,
                    void* cuda_stream);

/*
 * Packed-QKV across-heads RMSNorm + 3D RoPE + V copy (+ FP8 E4M3 output)
 * ("flashinfer.norm.fused_qk_rmsnorm_rope": summary, Parameters, Returns).
 *
 * Input row of token t: qkv[t] = [Q heads | K heads | V heads], each head
 * head_dim bf16 channels, (Hq + Hk + Hv) * head_dim per row, rows dense.
 *   Q: r = 1 / sqrt(sum over all Hq*head_dim channels of x^2 / (Hq*head_dim) + eps)
 *      y[c] = x[c] * r * q_weight[c]  (c < Hq*head_dim); K likewise over Hk*head_dim.
 *      With is_qk_norm == 0, y = x (weights and eps unused, may be NULL).
 *   Patch of token t: s = (t + pos_offset) mod (ppf*pph*ppw), row-major:
 *      f = s / (pph*ppw), h = (s / ppw) mod pph, w = s mod ppw.
 *   Pair slot j < head_dim/2 belongs to the frame axis for j < Cf/2, the height
 *      axis for the next Ch/2 slots, the width axis for the rest; with i the
 *      slot's index inside its axis group and C that group's channel count,
 *      theta_j = pos_axis * base^(-2i/C).
 *   Each Q and K head rotates its pairs: (2j, 2j+1) if interleave, else
 *      (j, j + head_dim/2) (NeoX), by theta_j as in qknr_rope_table.
 *   NeoX per axis (neox_per_axis = 1, interleave = 0): the page says only
 *      "NeoX-style" for interleave=False, which also reads as NeoX halves
 *      inside each axis group: with o the group's first channel and C its
 *      channel count, the pairs are (o + i, o + i + C/2), i < C/2, rotated by
 *      pos_axis * base^(-2i/C). The default (0) is the whole-head layout
 *      above; both give the same result for interleave == 1. This layout is
 *      built for channel groups that are multiples of 16 (else
 *      QKNR_ERR_UNSUPPORTED).
 *   Outputs: q_out [T, Hq, head_dim], k_out [T, Hk, head_dim], v_out
 *      [T, Hv, head_dim], dense. bf16; or with output_fp8, E4M3 of
 *      q*output_quant_scale, k*output_quant_scale and v*v_quant_scale.
 *      Without output_fp8, v_out is a bit copy of V.
 *   Range: the sums of squares are fp32, so a row whose Q or K sum of squares
 *      overflows fp32 (|x| above about 1e17 over 4096 channels) comes out as
 *      zeros or NaN; with eps == 0 an all-zero Q or K comes out as NaN (0/0).
 *
 * Validation: num_tokens divisible by ppf*pph*ppw for a whole call, any count
 * for a sequence shard (sequence_shard = 1); channel counts even,
 * non-negative, summing to head_dim; head_dim in {64, 128, 256}; heads >= 0 and
 * Hq + Hk + Hv >= 1; factor == 1 and attention_factor == 1 (YARN is not built:
 * QKNR_ERR_UNSUPPORTED); qkv and all outputs 16-byte aligned; no output
 * overlapping qkv or another output.
 */
typedef struct {
    size_t struct_size; /* sizeof(qknr_rope_3d_params); guards against ABI drift */
    const void* qkv;    /* bf16 [num_tokens, (Hq+Hk+Hv)*head_dim]               */
    const void* q_weight; /* bf16 [Hq*head_dim]                                   */
    const void* k_weight; /* bf16 [Hk*head_dim]                                   */
    void* q_out;        /* bf16 or E4M3 [num_tokens, Hq, head_dim]               */
    void* k_out;        /* bf16 or E4M3 [num_tokens, Hk, head_dim]               */
    void* v_out;        /* bf16 or E4M3 [num_tokens, Hv, head_dim]               */
    int64_t num_tokens;
    int64_t pos_offset; /* patch position of the first token (mod ppf*pph*ppw)   */
    int32_t ppf, pph, ppw;
    int32_t num_frame_channels, num_height_channels, num_width_channels;
    int32_t num_heads_q, num_heads_k, num_heads_v, head_dim;
    float eps;
    double base;         /* double: at large positions a float base shifts angles */
    int32_t interleave;  /* 1 = adjacent pairs (non-NeoX), 0 = NeoX half split   */
    float factor, low, high, attention_factor; /* YARN: only factor == 1 accepted */
    int32_t is_qk_norm;
    int32_t output_fp8;
    float output_quant_scale;
    float v_quant_scale;
    int32_t sequence_shard; /* 0: the whole patch sequence(s), num_tokens divisible
                               by ppf*pph*ppw; 1: a contiguous slice of a longer
                               sequence starting at patch position pos_offset
                               (one rank's part of a sharded call): any count */
    int32_t neox_per_axis;  /* NeoX pairs (interleave == 0) inside each axis group
                               instead of across the whole head; see below.
                               Ignored with interleave == 1. */
} qknr_rope_3d_params;

int qknr_rope_3d(const qknr_rope_3d_params* params, void* cuda_stream);

/*
 * Tensor-parallel 3D form. When the Q, K and V heads of a token are split
 * across ranks, each rank holds packed rows of its own heads only, but the
 * across-heads RMSNorm still covers all of Q's (and all of K's) channels on
 * every rank, not one rank's slice ("vllm_omni.diffusion.models.sana_wm.ucpe",
 * cam_prep_func, which leaves the norm to the model's own modules for exactly
 * this reason).
 * The transform is the one of qknr_rope_3d ("flashinfer.norm.
 * fused_qk_rmsnorm_rope"), split in two passes around one exchange:
 *
 *   1. qknr_rope_3d_partial_ssq: per token, the sums of x^2 over this call's
 *      Q channels and over its K channels -> ssq_out, fp32 [num_tokens][2].
 *      Only the Q and K part of each row is read; outputs, weights, eps and
 *      the FP8 fields of params are ignored (may be NULL / anything).
 *   2. the caller sums ssq_out over all ranks (an all-reduce).
 *   3. qknr_rope_3d_with_ssq: the full transform of this call's heads (RoPE,
 *      V copy, FP8 as usual) with r = 1 / sqrt(ssq[t][0] / (heads_q_total *
 *      head_dim) + eps) for Q and likewise for K over heads_k_total.
 *      params.is_qk_norm must be 1; heads_*_total >= this call's heads.
 *
 * With one rank (heads_*_total equal to the call's own heads) the passes give
 * the same result as qknr_rope_3d up to the order of the fp32 additions.
 * The [T][2] arrays are 8-byte aligned and must not overlap any other buffer.
 * Both passes run on the pipelined kernel: a row that does not fit two
 * buffers of shared memory returns QKNR_ERR_UNSUPPORTED.
 */
int qknr_rope_3d_partial_ssq(const qknr_rope_3d_params* params, float* ssq_out,
                             void* cuda_stream);
int qknr_rope_3d_with_ssq(const qknr_rope_3d_params* params, const float* ssq,
                          int32_t heads_q_total, int32_t heads_k_total, void* cuda_stream);

/*
 * UCPE camera prep ("vllm_omni.diffusion.models.sana_wm.ucpe": cam_prep_func).
 * The page lists the steps (ReLU, the K scale, the ray projection, RoPE) and
 * the shapes but no formula; the readings taken are these. For batch b, token
 * n, head h, with x the head_dim channels of that (b, n, h):
 *   Q: x' = max(x, 0); y = proj_q[b][n] applied to every block of four
 *      channels, y[4i'+i] = sum_j M[i][j] x'[4i'+j] (M row-major);
 *      out[2j]   = y[2j] c_j - y[2j+1] s_j,
 *      out[2j+1] = y[2j+1] c_j + y[2j] s_j,
 *      c_j = rope_cos[n][j], s_j = rope_sin[n][j], j < head_dim/2.
 *   K: k' = k_scale * max(x, 0); y = proj_kv[b][n] blockwise; rotated as Q.
 *      inflation_sq[b][h][n] = |y|^2 / |k'|^2, or 1 when k' is all zero.
 *   V: y = proj_kv[b][n] blockwise, not rotated.
 *   Outputs are stored transposed: q_trans[b][h][d][n] = out[d], likewise
 *   k_trans and v_trans; each value rounded once to act_dtype.
 * The definition of inflation_sq is not on the page (it names the output
 * only); this squared-norm gain of the key is a reading, as is which tensors
 * take ReLU and RoPE.
 *
 * act_dtype        QKNR_DT_BF16 or QKNR_DT_F16: q_normed, k_normed, v_raw and
 *                  the three outputs.
 * q_normed, k_normed, v_raw  [batch, num_tokens, num_heads, head_dim], dense,
 *                  read only (Q and K already RMS-normalised by the caller).
 * proj_q, proj_kv  float32 [batch, num_tokens, 4, 4], dense, row-major.
 * rope_cos, rope_sin  float32 [num_tokens, head_dim/2], dense, shared by the
 *                  batch.
 * q_trans, k_trans, v_trans  act_dtype [batch, num_heads, head_dim, num_tokens],
 *                  dense; written only. None may overlap an input or another
 *                  output (QKNR_ERR_ALIAS).
 * inflation_sq     float32 [batch, num_heads, num_tokens], or NULL to skip it.
 * head_dim         a multiple of 8 from 8 to 256; batch, num_tokens,
 *                  num_heads >= 0 (any of them 0: a no-op).
 * k_scale          any finite float (the page's value is
 *                  head_dim^-0.5 * spatial_tokens^-0.5).
 * Alignment: every pointer 16-byte aligned (QKNR_ERR_ALIGN otherwise).
 * Any num_tokens is allowed; a multiple of 16 is fastest (every output row
 * then starts on a 32-byte sector: about 7% slower at 8 mod 16, 38% at counts
 * that are not multiples of 8, at head_dim 112). Kernels: with at least two heads, head_dim
 * 72..120, device-memory q/k/v and batch*num_tokens >= 64, a warp-specialised
 * pipelined kernel (any num_tokens); else, with at least two heads,
 * head_dim <= 128 and an even num_tokens, a barrier-synchronised pipelined
 * kernel; else a general one, which writes two bytes at a time when
 * num_tokens is not a multiple of 8 and, when there are enough 64-token tiles
 * to fill the GPU, takes whole tiles with all their heads per CTA.
 * Range: every kernel applies k_scale to K's rotated result (the projection
 * and the rotation are linear) and take the two fp32 sums of squares over the
 * unscaled ReLU key, so the scale itself never underflows or overflows them.
 * A key whose squares all underflow fp32 (every channel below about 1e-19 in
 * magnitude) counts as a zero key (inflation_sq 1); a key whose sum of
 * squares overflows fp32 (channels above about 1e18 at head_dim 256, 1.8e19
 * for one channel) gives inflation_sq NaN, where the fp64 definition stays
 * finite.
 * The warp-specialised kernel's waits (its compute warps on the copy warp's
 * ring stages, the copy warp on the compute warps) are bounded at 2 s; on
 * expiry the launch abandons its remaining steps and raises bit 0 of the
 * device status word (qknr_device_status). The other two kernels wait only on
 * their own cp.async groups and CTA barriers, which always complete.
 */
int qknr_ucpe_cam_prep(const void* q_normed, const void* k_normed, const void* v_raw,
                       const float* proj_q, const float* proj_kv, const float* rope_cos,
                       const float* rope_sin, void* q_trans, void* k_trans, void* v_trans,
                       float* inflation_sq, int32_t act_dtype, int64_t batch,
                       int64_t num_tokens, int32_t num_heads, int32_t head_dim, float k_scale,
                       void* cuda_stream);

/*
 * Device-side status of this library's kernels on the current device, for
 * failures that can only be seen on the GPU. Bit 0: a kernel's wait on one of
 * its own bulk copies (or, in the camera prep, on another warp of its CTA) ran
 * past its time limit (2 s), so that launch abandoned
 * its remaining tokens and its outputs are incomplete; the kernel still ended
 * normally and the CUDA context stays usable. The word accumulates over
 * launches until cleared. Unlike every other entry point this one
 * synchronises: it reads the word after the work already queued on
 * `cuda_stream`, then clears it if `clear` is non-zero.
 */
int qknr_device_status(void* cuda_stream, uint32_t* status_out, int32_t clear);

/*
 * Test hook for the timeout path above (not for production use). While
 * extra_bytes is non-zero, every later launch of a bulk-copy kernel (3D and
 * table forms, the camera prep's warp-specialised kernel) on any thread makes each
 * ring buffer wait for extra_bytes more
 * than its copy delivers, so its waits
 * run out after limit_ns and the launch takes the abandon path; the copies
 * themselves complete, so nothing is left in flight. extra_bytes == 0 turns
 * the hook off (limit_ns is then ignored and the 2 s limit returns).
 */
int qknr_test_set_wait_fault(uint32_t extra_bytes, uint64_t limit_ns);

/* Static text for a status code. */
const char* qknr_status_string(int status);

/* Text on the last failing call of this host thread ("" if none). */
const char* qknr_last_error_detail(void);

/* QKNR_ABI_VERSION of the built library. */
int qknr_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QKNR_H_ */
