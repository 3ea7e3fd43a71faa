// UCPE camera prep, the transform that vLLM-Omni's SANA-WM UCPE page
// ("vllm_omni.diffusion.models.sana_wm.ucpe", cam_prep_func) applies on the
// camera branch before its linear attention. For every token n and head h of
// camera Q, K, V laid out [B, N, H, D]:
//   Q: ReLU, then every block of four channels times the token's 4x4 proj_q,
//      then RoPE on adjacent channel pairs (2j, 2j+1) with cos/sin column j of
//      row n of the [N, D/2] tables;
//   K: ReLU, times k_scale, times proj_kv blockwise, RoPE; and inflation_sq,
//      the squared-norm gain |proj_kv k'|^2 / |k'|^2 of the scaled key (1 for a
//      zero key);
//   V: times proj_kv blockwise;
// and the three results are stored transposed, [B, H, D, N].
//
// The work is a stream over HBM (about 1.5 flops per byte). Three kernels do
// it, all built for coalescing on both sides of the transpose:
// ucpe_fast_kernel (warp-specialised, further down) for head_dim 72..120 with
// at least two heads; ucpe_sync_kernel (barrier-synchronised) for the other
// head_dims up to 128 with an even token count and at least two heads; and
// ucpe_prep_kernel for every other shape. The general kernel:
//   - work unit: a tile of 64 consecutive tokens of one (batch, head), units
//     numbered with the head fastest, so that the units in flight at once
//     share their tokens' cos/sin rows and matrices in L2; or, when there are
//     enough tiles to give every CTA whole tiles (TILE_MAJOR), a tile with
//     all its heads in turn, its matrices and cos/sin rows staged once
//     (56.6 against 48.5% of HBM at head_dim 256, 8 heads);
//   - a thread takes four tokens of one 8-channel chunk (two projection
//     blocks, four rotation pairs). Consecutive threads read consecutive
//     16-byte chunks of a token's row, so each warp load covers whole rows;
//   - results go to a transposed staging tile in shared memory, [D][64] per
//     tensor, as 8-byte words (one channel of the thread's four tokens); the
//     16-byte chunks of each row are XOR-swizzled by (d / 8) mod 8, so that
//     the writers of one token's chunks land in different banks while a row
//     still reads back as eight whole chunks;
//   - the tile leaves with 16-byte stores, eight threads per output row: each
//     row's 64 tokens are one 128-byte line of the [B, H, D, N] output.
// The 4x4 matrices and the cos/sin rows of the tile's tokens are copied into
// shared memory with cp.async (the next tile's while this one's results leave);
// the per-chunk key sums are added per token in a fixed order, so the results
// do not depend on the launch shape.
#include "common.cuh"
#include "ucpe_launch.h"
#include "launch_cache.h"

#include <cuda.h>  // CUtensorMap and its encoding (through the runtime's driver entry point)

#include <algorithm>
#include <mutex>

namespace qknr {
namespace {

constexpr int kTile = 64;        // tokens per tile (one 128-byte output row)
constexpr int kPairs = kTile / 2;
constexpr int kProjStride = 36;  // floats per token in the staged matrices (32 used)

// Threads per CTA: one per (4-token group, 8-channel chunk) of a tile.
int ucpe_block(int D) { return ((kTile / 4) * (D / 8) + 31) / 32 * 32; }

int ucpe_smem(int D) {
    return 3 * D * kTile * 2 + kTile * kProjStride * 4 + 2 * kTile * (D / 2) * 4 +
           kTile * (D / 8) * 8;
}

// Byte offset of (channel d, tile token t) inside one tensor's staging tile.
__device__ __forceinline__ int stage_offset(int d, int t) {
    return d * (kTile * 2) + ((((t >> 3) ^ (d >> 3)) & 7) << 4) + ((t & 7) << 1);
}

// y = m x for one block of four channels, m row-major in shared memory.
__device__ __forceinline__ void project_block(const float* m, const float* x, float* y) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 r = *reinterpret_cast<const float4*>(m + 4 * i);
        y[i] = fmaf(r.w, x[3], fmaf(r.z, x[2], fmaf(r.y, x[1], r.x * x[0])));
    }
}

// 16-byte asynchronous copy global -> shared; with valid == false the 16
// bytes are zero-filled and nothing is read.
__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst_smem)),
                 "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

// 4-byte asynchronous copy global -> shared; with valid == false the 4 bytes
// are zero-filled and nothing is read.
__device__ __forceinline__ void cp_async4(void* dst_smem, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst_smem)),
                 "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}

__device__ __forceinline__ void st_u16(void* p, uint16_t v) {
    asm volatile("st.global.u16 [%0], %1;" ::"l"(p), "h"(v) : "memory");
}

// max(x, 0) on both 16-bit halves of a word.
template <bool H16>
__device__ __forceinline__ uint32_t relu2(uint32_t w) {
    if constexpr (H16) {
        __half2 h = __hmax2(*reinterpret_cast<const __half2*>(&w), __float2half2_rn(0.0f));
        return *reinterpret_cast<uint32_t*>(&h);
    } else {
        __nv_bfloat162 h = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&w),
                                   __float2bfloat162_rn(0.0f));
        return *reinterpret_cast<uint32_t*>(&h);
    }
}

// Channels 2e and 2e+1 of a token pair: (lower-channel value of token A, of
// token B) and the same for the upper channel.
template <bool H16>
__device__ __forceinline__ void widen_pair(uint32_t wa, uint32_t wb, float2& lo, float2& hi) {
    if constexpr (H16) {
        const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&wa));
        const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&wb));
        lo = make_float2(fa.x, fb.x);
        hi = make_float2(fa.y, fb.y);
    } else {
        lo = make_float2(bf16_lo(wa), bf16_lo(wb));
        hi = make_float2(bf16_hi(wa), bf16_hi(wb));
    }
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// The tile's per-token inputs that every head shares, copied asynchronously
// into shared memory: the two 4x4 matrices ([kTile][kProjStride] floats,
// proj_q then proj_kv) and the cos and sin rows ([kTile][D/2] floats each).
__device__ __forceinline__ void stage_token_inputs(const UcpeArgs& a, int64_t b, int64_t n0,
                                                   int tv, int tid, int nthr, float* proj,
                                                   float* cosr, float* sinr) {
    for (int f = tid; f < kTile * 8; f += nthr) {
        const int t = f >> 3, r = f & 7;
        const bool ok = t < tv;
        const float* src = (r < 4 ? a.proj_q : a.proj_kv) +
                           (ok ? (b * a.num_tokens + n0 + t) * 16 + (r & 3) * 4 : 0);
        cp_async16(proj + t * kProjStride + r * 4, src, ok);
    }
    const int q4 = a.head_dim / 8;  // float4 per token row of a table
    for (int f = tid; f < kTile * q4 * 2; f += nthr) {
        const int which = f >= kTile * q4;  // 0: cos, 1: sin
        const int g = f - which * kTile * q4;
        const int t = g / q4, k4 = g - (g / q4) * q4;
        const bool ok = t < tv;
        const float* src = (which ? a.rope_sin : a.rope_cos) +
                           (ok ? (n0 + t) * (a.head_dim / 2) + 4 * k4 : 0);
        cp_async16((which ? sinr : cosr) + g * 4, src, ok);
    }
    cp_async_commit();
}

// Q, K and V chunks of four tokens (one item), held in registers.
__device__ __forceinline__ void load_item(const UcpeArgs& a, int64_t b, int64_t n0, int h, int tv,
                                          int p, int c, uint4 (&raw)[3][4]) {
    const int D = a.head_dim;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int t = 4 * p + u;
        if (t < tv) {
            const int64_t row = ((b * a.num_tokens + n0 + t) * a.heads + h) * D + 8 * c;
            raw[0][u] = ld_nc_v4(a.q + row * 2);
            raw[1][u] = ld_nc_v4(a.k + row * 2);
            raw[2][u] = ld_nc_v4(a.v + row * 2);
        } else {
            raw[0][u] = raw[1][u] = raw[2][u] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

// One token's 8 channels of tensor X (0 = Q, 1 = K, 2 = V): element steps,
// projection, rotation; for K also the two sums of squares.
template <bool H16, int X>
__device__ __forceinline__ void transform8(const uint4& raw, const float* m, const float* cr,
                                           const float* sr, float k_scale, float* y, float& si,
                                           float& so) {
    float x[8];
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = act2_to_f2<H16>(w[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
    if (X < 2) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = fmaxf(x[e], 0.0f);
    }
    project_block(m, x, y);
    project_block(m, x + 4, y + 4);
    if (X == 1) {
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            a = fmaf(x[e], x[e], a);
            b = fmaf(y[e], y[e], b);
        }
        si = a;
        so = b;
    }
    if (X < 2) {
        const float4 cs = *reinterpret_cast<const float4*>(cr);
        const float4 sn = *reinterpret_cast<const float4*>(sr);
        const float cj[4] = {cs.x, cs.y, cs.z, cs.w};
        const float sj[4] = {sn.x, sn.y, sn.z, sn.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float ya = y[2 * j], yb = y[2 * j + 1];
            y[2 * j] = fmaf(ya, cj[j], -yb * sj[j]);
            y[2 * j + 1] = fmaf(yb, cj[j], ya * sj[j]);
        }
    }
    // K's scale goes on the rotated result: the projection and the rotation
    // are linear, and the sums above are of the unscaled key, whose gain is
    // the scaled key's (no underflow or overflow from the scale in them).
    if (X == 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] *= k_scale;
    }
}

// Tensor X of the item: four tokens, results packed two tokens to a word (the
// lower token in the low half) and written to the staging tile as one 8-byte
// word per channel.
template <bool H16, int X>
__device__ __forceinline__ void item_tensor(const uint4 (&raw)[3][4], const float* proj,
                                            const float* cosr, const float* sinr, int D, int p,
                                            int c, float k_scale, unsigned char* tile_x,
                                            float* si, float* so) {
    uint32_t packed[8][2];
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
        float y0[8], y1[8];
        const int u0 = 2 * pr, u1 = 2 * pr + 1;
        const int t0 = 4 * p + u0, t1 = 4 * p + u1;
        const int moff = X == 0 ? 0 : 16;
        const int roff = 4 * c;
        transform8<H16, X>(raw[X][u0], proj + t0 * kProjStride + moff, cosr + t0 * (D / 2) + roff,
                           sinr + t0 * (D / 2) + roff, k_scale, y0, si[u0], so[u0]);
        transform8<H16, X>(raw[X][u1], proj + t1 * kProjStride + moff, cosr + t1 * (D / 2) + roff,
                           sinr + t1 * (D / 2) + roff, k_scale, y1, si[u1], so[u1]);
#pragma unroll
        for (int e = 0; e < 8; ++e) packed[e][pr] = f2_to_act2<H16>(make_float2(y0[e], y1[e]));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        *reinterpret_cast<uint2*>(tile_x + stage_offset(8 * c + e, 4 * p)) =
            make_uint2(packed[e][0], packed[e][1]);
    }
}

// Position of a tile in the (batch, token tile, head) order, head fastest,
// advanced by a fixed stride without divisions.
struct TileCursor {
    int64_t b, tn;
    int h;
    __device__ __forceinline__ void advance(int64_t step_bt, int step_h, int H, int64_t tiles_n) {
        h += step_h;
        int64_t dbt = step_bt;
        if (h >= H) {
            h -= H;
            ++dbt;
        }
        tn += dbt;
        while (tn >= tiles_n) {
            tn -= tiles_n;
            ++b;
        }
    }
};

template <bool H16, bool TILE_MAJOR>
__global__ void __launch_bounds__(512) ucpe_prep_kernel(const UcpeArgs a) {
    const int D = a.head_dim, C = D / 8, H = a.heads;
    const int64_t N = a.num_tokens;
    const int64_t tiles_n = (N + kTile - 1) / kTile;
    // TILE_MAJOR: a CTA takes whole tiles and their heads in turn, staging the
    // tile's matrices and cos/sin rows once; otherwise single (tile, head)
    // units, the head fastest.
    const int64_t nunits = a.batch * tiles_n * (TILE_MAJOR ? 1 : H);
    const int tid = threadIdx.x, nthr = blockDim.x;
    const bool vec_out = (N & 7) == 0;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* stage = smem;  // [3][D][kTile] 16-bit, swizzled rows
    float* proj = reinterpret_cast<float*>(smem + 3 * D * kTile * 2);  // [kTile][kProjStride]
    float* cosr = proj + kTile * kProjStride;                            // [kTile][D/2]
    float* sinr = cosr + kTile * (D / 2);                                // [kTile][D/2]
    float2* part = reinterpret_cast<float2*>(sinr + kTile * (D / 2));   // [kTile][C]

    // This thread's item: tokens 4p..4p+3 of the tile, channels 8c..8c+7.
    const int p = tid / C, c = tid - (tid / C) * C;
    const bool has_item = tid < (kTile / 4) * C;

    int64_t unit = blockIdx.x;
    if (unit >= nunits) return;
    TileCursor cur;
    int64_t step_bt = 0;
    int step_h = 0;
    if constexpr (TILE_MAJOR) {
        cur.h = 0;
        cur.tn = unit;
    } else {
        step_bt = (int64_t)gridDim.x / H;
        step_h = (int)((int64_t)gridDim.x - step_bt * H);
        cur.h = (int)(unit % H);
        cur.tn = unit / H;
    }
    cur.b = cur.tn / tiles_n;
    cur.tn -= cur.b * tiles_n;

    griddep_wait();
    griddep_launch_dependents();

    // Prologue: the first tile's inputs.
    uint4 raw[3][4];
    {
        const int64_t n0 = cur.tn * kTile;
        const int tv = (int)min((int64_t)kTile, N - n0);
        stage_token_inputs(a, cur.b, n0, tv, tid, nthr, proj, cosr, sinr);
        if (has_item) load_item(a, cur.b, n0, cur.h, tv, p, c, raw);
        cp_async_wait_all();
    }
    __syncthreads();

    while (true) {
        const int64_t b = cur.b, n0 = cur.tn * kTile;
        const int h = cur.h;
        const int tv = (int)min((int64_t)kTile, N - n0);

        if (has_item) {
            float si[4], so[4];
            item_tensor<H16, 0>(raw, proj, cosr, sinr, D, p, c, a.k_scale, stage, si, so);
            item_tensor<H16, 1>(raw, proj, cosr, sinr, D, p, c, a.k_scale, stage + D * kTile * 2,
                                si, so);
            item_tensor<H16, 2>(raw, proj, cosr, sinr, D, p, c, a.k_scale,
                                stage + 2 * D * kTile * 2, si, so);
#pragma unroll
            for (int u = 0; u < 4; ++u) part[(4 * p + u) * C + c] = make_float2(si[u], so[u]);
        }
        __syncthreads();

        // The next unit's inputs go out before this one's stores; the tile's
        // matrices and cos/sin rows only when the tile changes.
        bool more, new_tile = true;
        if constexpr (TILE_MAJOR) {
            if (cur.h + 1 < H) {
                ++cur.h;
                more = true;
                new_tile = false;
            } else {
                unit += gridDim.x;
                more = unit < nunits;
                if (more) {
                    cur.h = 0;
                    cur.advance(gridDim.x, 0, 1, tiles_n);
                }
            }
        } else {
            unit += gridDim.x;
            more = unit < nunits;
            if (more) cur.advance(step_bt, step_h, H, tiles_n);
        }
        if (more) {
            const int64_t nn0 = cur.tn * kTile;
            const int ntv = (int)min((int64_t)kTile, N - nn0);
            if (new_tile) stage_token_inputs(a, cur.b, nn0, ntv, tid, nthr, proj, cosr, sinr);
            if (has_item) load_item(a, cur.b, nn0, cur.h, ntv, p, c, raw);
        }

        // The staged tile leaves as whole 128-byte output rows.
        const int64_t out_head = (b * H + h) * (int64_t)D;
#pragma unroll
        for (int X = 0; X < 3; ++X) {
            uint8_t* out = X == 0 ? a.q_out : (X == 1 ? a.k_out : a.v_out);
            const unsigned char* tile_x = stage + X * D * kTile * 2;
            for (int i = tid; i < D * 8; i += nthr) {
                const int d = i >> 3, j = i & 7;
                const uint4 val = *reinterpret_cast<const uint4*>(
                    tile_x + d * (kTile * 2) + (((j ^ (d >> 3)) & 7) << 4));
                const int64_t n = n0 + 8 * j;
                uint8_t* dst = out + ((out_head + d) * N + n) * 2;
                if (vec_out && n + 8 <= N) {
                    st_v4(dst, val);
                } else {
                    const uint32_t w[4] = {val.x, val.y, val.z, val.w};
                    for (int e = 0; e < 8 && n + e < N; ++e)
                        reinterpret_cast<uint16_t*>(dst)[e] =
                            (uint16_t)(w[e >> 1] >> ((e & 1) * 16));
                }
            }
        }
        if (a.inflation_sq) {
            for (int t = tid; t < tv; t += nthr) {
                float si = 0.f, so = 0.f;
                for (int cc = 0; cc < C; ++cc) {
                    const float2 v = part[t * C + cc];
                    si += v.x;
                    so += v.y;
                }
                a.inflation_sq[(b * H + h) * N + n0 + t] =
                    (si > 0.f && a.k_scale != 0.0f) ? so / si : 1.0f;
            }
        }
        if (!more) break;
        cp_async_wait_all();
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Warp-specialised pipelined kernel: head_dim 72..120, any token count, at
// least two heads, q/k/v in device memory, at least 64 rows.
//
// Work unit: a step is one head of a tile of 64 tokens of one batch element;
// a CTA takes its tiles in turn and each tile's heads in order. The CTA is D/8
// compute warps and one copy warp:
//   - the copy warp's lane 0 brings each step's Q, K and V rows (64 tokens,
//     fast_row_elems(D) channels from the head's first) into a stage of a
//     shared-memory ring with one 2D tensor copy per tensor, counted in bytes
//     on the stage's "full" mbarrier, STAGES - 1 steps ahead. (One bulk copy
//     per row measured 2.6x slower: the copy engine took about 27 such small
//     copies per microsecond per SM, below what 192 rows per step need.)
//     Before refilling a stage it waits on the stage's "empty" mbarrier, which
//     every compute thread arrives on once it has read the stage. At a tile's
//     first step it also writes the tile's two 4x4 matrices into shared
//     memory, interleaved by the token pairs the compute lanes own
//     (double-buffered per tile, with their own full/empty mbarriers), and it
//     adds up the key sums of finished steps and writes inflation_sq;
//   - lane i of compute warp w owns the tokens i and i + 32 of the tile and
//     the 8-channel chunk w. Per step it widens, projects, rotates and rounds
//     its two tokens x eight channels of each tensor with packed fp32x2
//     instructions (the tile's cos/sin values sit in registers for all its
//     heads) and stores 16-bit values straight to [B, H, D, N]: the 32 lanes
//     of a warp write the two 64-byte halves of a 128-byte output row, so any
//     token count works. When num_tokens is 8 mod 16 (rows 16 bytes off a
//     32-byte sector) the warp instead writes its 8 x 64 results into its own
//     1 KB shared buffer and sends whole rows as 16-byte stores. Its key sums
//     go to a double-buffered shared array for the copy warp.
// No CTA-wide barrier: compute warps wait only for their data, so a slow warp
// delays the others only when the ring runs dry. Every wait is bounded in
// time; on expiry the waiter raises the CTA's abort flag and bit 0 of the
// device status word, every other wait gives up at the flag, and the copy
// warp waits for its own copies (which always land) before the CTA ends.
// Padding: a stage row is an odd number of 16-byte chunks (fast_row_elems),
// so that the chunk c of eight consecutive rows falls in distinct bank groups;
// a token pair's interleaved matrices take 144 bytes for the same reason.
constexpr int kFastMaxD = 128;  // the barrier-synchronised kernel's limit
constexpr int kWsMaxD = 120;    // the warp-specialised kernel's (16 warps of 32 threads)
constexpr int kMatStride = 36;  // floats per token pair per matrix (32 used)

// Tensor maps of q, k and v as 2D tensors [batch * num_tokens rows,
// heads * head_dim columns] of 16-bit elements, box [64 rows,
// fast_row_elems(D) columns], no swizzle, zeros past the edges.
struct UcpeMaps {
    CUtensorMap m[3];
};

// Bytes per token row in a ring stage: D channels and 8 more when D/8 is even,
// so that the row is an odd number of 16-byte chunks and the chunk c of eight
// consecutive rows falls in eight distinct bank groups. (The copies fill the
// extra channels with the next head's, or with zeros past the last head.)
__host__ __device__ inline int fast_row_elems(int D) { return ((D / 8) & 1) ? D : D + 8; }
__host__ __device__ inline int fast_row_pitch(int D) { return 2 * fast_row_elems(D); }
__host__ __device__ inline int fast_stage_bytes(int D) { return 3 * kTile * fast_row_pitch(D); }

struct FastLayout {
    int ring, out, mats, part, bars, abort, total, stages;
};

// The ring, the compute warps' 1 KB output buffers (staged), two matrix
// buffers, two key-sum buffers, the mbarriers
// (full[STAGES], empty[STAGES], mats_full[2], mats_empty[2], sums_full[2],
// sums_empty[2]) and the abort flag.
__host__ __device__ inline FastLayout fast_layout(int D, int stages, bool staged) {
    FastLayout L;
    const int C = D / 8;
    L.stages = stages;
    L.ring = 0;
    L.out = stages * fast_stage_bytes(D);               // [C][8][kTile] 16-bit
    L.mats = L.out + (staged ? C * 8 * kTile * 2 : 0);  // [2][2][32][kMatStride] f32
    L.part = L.mats + 2 * 2 * kPairs * kMatStride * 4;  // [2][C][64] float2
    L.bars = L.part + 2 * C * kTile * 8;
    L.abort = L.bars + (2 * stages + 8) * 8;
    L.total = L.abort + 16;
    return L;
}

__device__ unsigned int g_ucpe_status;

// A step of this CTA: head h of its ti-th tile (tile blockIdx.x + ti * grid),
// advanced one head at a time (the division runs once per tile).
struct FastStep {
    int64_t ti, b, n0;
    int h, tv;
    bool valid;

    __device__ __forceinline__ void locate(const UcpeArgs& a, int64_t tiles_n, int64_t ntiles) {
        const int64_t tile = blockIdx.x + ti * (int64_t)gridDim.x;
        valid = tile < ntiles;
        b = valid ? tile / tiles_n : 0;
        n0 = valid ? (tile - b * tiles_n) * kTile : 0;
        tv = valid ? (int)min((int64_t)kTile, a.num_tokens - n0) : 0;
    }
    __device__ __forceinline__ void next(const UcpeArgs& a, int64_t tiles_n, int64_t ntiles) {
        if (++h == a.heads) {
            h = 0;
            ++ti;
            locate(a, tiles_n, ntiles);
        }
    }
};

// Copy warp: the tile's matrices into matrix buffer `mats`, interleaved by the
// token pairs (i, i + 32) a compute lane owns (plain loads and shared stores;
// only the tile's tokens).
__device__ __forceinline__ void fast_stage_mats(const UcpeArgs& a, const FastStep& st, float* mats,
                                                int lane) {
    for (int f = lane; f < st.tv * 8; f += 32) {
        const int t = f >> 3, r = f & 7;  // token, float4 r of its two matrices
        const float4 v = __ldg(reinterpret_cast<const float4*>(
            (r < 4 ? a.proj_q : a.proj_kv) + (st.b * a.num_tokens + st.n0 + t) * 16) + (r & 3));
        float* d = mats + ((r >> 2) * kPairs + (t & 31)) * kMatStride + (r & 3) * 8 + (t >> 5);
        d[0] = v.x;
        d[2] = v.y;
        d[4] = v.z;
        d[6] = v.w;
    }
}

// Copy warp, lane 0: one step's Q, K and V rows (64 tokens from the tile's
// first, fast_row_elems(D) channels from head h's first) into ring stage
// `buf`, one tensor copy per tensor, counted in bytes on `full`. Rows past the
// end of the tensor arrive as zeros.
__device__ __forceinline__ void fast_stage_rows(const CUtensorMap* maps, const UcpeArgs& a,
                                                const FastStep& st, unsigned char* buf,
                                                uint64_t* full) {
    const int x = st.h * a.head_dim;                  // a multiple of 8 elements: 16 bytes
    const int y = (int)(st.b * a.num_tokens + st.n0);
    const int tensor_bytes = kTile * fast_row_pitch(a.head_dim);
#pragma unroll
    for (int X = 0; X < 3; ++X) {
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3}], [%4];"
            ::"r"(smem_u32(buf + X * tensor_bytes)), "l"(reinterpret_cast<uint64_t>(&maps[X])),
              "r"(x), "r"(y), "r"(smem_u32(full))
            : "memory");
    }
}

// Copy warp: inflation_sq of step r (tile st, head st.h) from the compute
// warps' key sums in key-sum buffer r & 1, then that buffer is free again.
__device__ __forceinline__ bool fast_reduce_sums(const UcpeArgs& a, const FastStep& st, int64_t r,
                                                 const float2* part, uint64_t* sums_full,
                                                 uint64_t* sums_empty, int C, int lane,
                                                 uint64_t limit, volatile uint32_t* abort_flag) {
    const int p = (int)(r & 1);
    if (!mbar_wait_abortable(&sums_full[p], (uint32_t)((r >> 1) & 1), limit, abort_flag))
        return false;
    if (a.inflation_sq) {
        const float2* pr = part + p * C * kTile;
        const bool key_scaled = a.k_scale != 0.0f;
        for (int t = lane; t < st.tv; t += 32) {
            float s_in = 0.f, s_out = 0.f;
            for (int cc = 0; cc < C; ++cc) {
                const float2 v = pr[cc * kTile + t];
                s_in += v.x;
                s_out += v.y;
            }
            a.inflation_sq[(st.b * a.heads + st.h) * a.num_tokens + st.n0 + t] =
                (s_in > 0.f && key_scaled) ? s_out / s_in : 1.0f;
        }
    }
    mbar_arrive(&sums_empty[p]);
    return true;
}

// Tensor X of this thread's tokens (i, i + 32) and chunk c: widen, ReLU (Q,
// K), project, rotate (Q, K), scale (K), round; each channel's two results are
// stored straight to the output as 16-bit values (the 32 lanes of a warp write
// the 64-byte halves of one 128-byte output row), each only if its token is in
// the tile (va, vb). STAGED: the warp's 8 x 64 results go through its 1 KB
// buffer obuf instead and leave as 16-byte stores of whole rows (tokens past
// tv left out). For K, the two tokens' sums of squares go to si/so.
template <bool H16, int X, bool STAGED>
__device__ __forceinline__ void fast_tensor(const unsigned char* in, const float* mats,
                                            const float2 (&cj)[4], const float2 (&sj)[4],
                                            int pitch, int i, int c, float k_scale,
                                            uint8_t* out_row0, int64_t row_bytes, bool va, bool vb,
                                            float2& si, float2& so, unsigned char* obuf, int tv) {
    const unsigned char* r0 = in + (X * kTile + i) * pitch + 16 * c;
    const uint4 ra = *reinterpret_cast<const uint4*>(r0);
    const uint4 rb = *reinterpret_cast<const uint4*>(r0 + kPairs * pitch);
    uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
    uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
    if (X < 2) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            wa[e] = relu2<H16>(wa[e]);
            wb[e] = relu2<H16>(wb[e]);
        }
    }
    float2 x[8], y[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) widen_pair<H16>(wa[e], wb[e], x[2 * e], x[2 * e + 1]);
    const float* m = mats + ((X == 0 ? 0 : kPairs) + i) * kMatStride;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 r01 = *reinterpret_cast<const float4*>(m + 8 * i);
        const float4 r23 = *reinterpret_cast<const float4*>(m + 8 * i + 4);
        const float2 m0 = make_float2(r01.x, r01.y), m1 = make_float2(r01.z, r01.w);
        const float2 m2 = make_float2(r23.x, r23.y), m3 = make_float2(r23.z, r23.w);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            const float2* xb = x + 4 * blk;
            y[4 * blk + i] = fma2(m3, xb[3], fma2(m2, xb[2], fma2(m1, xb[1], mul2(m0, xb[0]))));
        }
    }
    if (X == 1) {
        float2 a2 = make_float2(0.f, 0.f), b2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            a2 = fma2(x[e], x[e], a2);
            b2 = fma2(y[e], y[e], b2);
        }
        si = a2;
        so = b2;
    }
    if (X < 2) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 ya = y[2 * j], yb = y[2 * j + 1];
            const float2 bs = mul2(yb, sj[j]);
            y[2 * j] = fma2(ya, cj[j], make_float2(-bs.x, -bs.y));
            y[2 * j + 1] = fma2(yb, cj[j], mul2(ya, sj[j]));
        }
    }
    if (X == 1) {
        const float2 ks = make_float2(k_scale, k_scale);
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = mul2(y[e], ks);
    }
    if constexpr (STAGED) {
        const uint32_t sb = smem_u32(obuf);
        __syncwarp();  // the warp has read back the previous tensor's tile
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t w = f2_to_act2<H16>(y[e]);
            asm volatile("st.shared.u16 [%0], %1;" ::"r"(sb + e * 2 * kTile + 2 * i),
                         "h"((uint16_t)w)
                         : "memory");
            asm volatile("st.shared.u16 [%0], %1;" ::"r"(sb + e * 2 * kTile + 2 * kPairs + 2 * i),
                         "h"((uint16_t)(w >> 16))
                         : "memory");
        }
        __syncwarp();
        const int q = i & 7;  // 16-byte chunk q (tokens 8q..8q+7) of rows i/8 and i/8 + 4
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int r = (i >> 3) + 4 * hf;
            uint4 v;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(sb + r * 2 * kTile + 16 * q)
                         : "memory");
            uint8_t* dst = out_row0 + (int64_t)r * row_bytes + 16 * q;
            if (8 * q + 8 <= tv) {
                st_v4(dst, v);
            } else {
                const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
                for (int t = 0; t < 8 && 8 * q + t < tv; ++t)
                    st_u16(dst + 2 * t, (uint16_t)(ww[t >> 1] >> ((t & 1) * 16)));
            }
        }
    } else {
        uint8_t* o = out_row0 + 2 * i;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t w = f2_to_act2<H16>(y[e]);
            if (va) st_u16(o + (int64_t)e * row_bytes, (uint16_t)w);
            if (vb) st_u16(o + (int64_t)e * row_bytes + 2 * kPairs, (uint16_t)(w >> 16));
        }
    }
}

// At most 15 compute warps (head_dim <= 120) and the copy warp: four warps per
// scheduler, which leaves 128 registers a thread.
template <bool H16, int STAGES, bool STAGED>
__global__ void __launch_bounds__(512, 1)
    ucpe_fast_kernel(const UcpeArgs a, const __grid_constant__ UcpeMaps maps,
                     const UcpeControl ctl) {
    const int D = a.head_dim, C = D / 8, H = a.heads;
    const int64_t N = a.num_tokens;
    const int64_t tiles_n = (N + kTile - 1) / kTile;
    const int64_t ntiles = a.batch * tiles_n;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const FastLayout L = fast_layout(D, STAGES, STAGED);

    extern __shared__ __align__(128) unsigned char smem[];
    float2* part = reinterpret_cast<float2*>(smem + L.part);  // [2][C][64]
    float* mats_base = reinterpret_cast<float*>(smem + L.mats);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);  // [STAGES]: copy warp, bytes
    uint64_t* empty = full + STAGES;          // [STAGES]: every compute thread
    uint64_t* mats_full = empty + STAGES;     // [2]: the copy warp's lanes
    uint64_t* mats_empty = mats_full + 2;     // [2]: every compute thread
    uint64_t* sums_full = mats_full + 4;      // [2]: every compute thread
    uint64_t* sums_empty = mats_full + 6;     // [2]: the copy warp's lanes
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L.abort);

    if ((int64_t)blockIdx.x >= ntiles) return;
    // this CTA's steps: its tiles x heads
    const int64_t my_tiles = (ntiles - 1 - blockIdx.x) / gridDim.x + 1;
    const int64_t nsteps = my_tiles * H;
    const int consumers = 32 * C;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], consumers);
        }
        for (int p = 0; p < 2; ++p) {
            mbar_init(&mats_full[p], 32);
            mbar_init(&mats_empty[p], consumers);
            mbar_init(&sums_full[p], consumers);
            mbar_init(&sums_empty[p], 32);
        }
        *abort_flag = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();
    griddep_launch_dependents();

    bool ok = true;
    if (warp == C) {
        // ------------------------------- copy warp -------------------------------
        FastStep st{}, rd{};  // the step to issue; the step whose key sums are next
        st.locate(a, tiles_n, ntiles);
        rd = st;
        int64_t s = 0, reduced = 0;
        for (; s < nsteps; ++s) {
            const int slot = (int)(s % STAGES);
            if (s >= STAGES) {
                // the compute warps are done with step s - STAGES: its stage is
                // free and its key sums are (being) written
                ok = mbar_wait_abortable(&empty[slot], (uint32_t)((s / STAGES - 1) & 1),
                                         ctl.wait_limit_ns, abort_flag);
                if (!ok) break;
                ok = fast_reduce_sums(a, rd, reduced, part, sums_full, sums_empty, C, lane,
                                      ctl.wait_limit_ns, abort_flag);
                if (!ok) break;
                ++reduced;
                rd.next(a, tiles_n, ntiles);
            }
            if (st.h == 0) {
                const int m = (int)(st.ti & 1);
                if (st.ti >= 2) {
                    ok = mbar_wait_abortable(&mats_empty[m], (uint32_t)((st.ti / 2 - 1) & 1),
                                             ctl.wait_limit_ns, abort_flag);
                    if (!ok) break;
                }
                fast_stage_mats(a, st, mats_base + m * 2 * kPairs * kMatStride, lane);
                mbar_arrive(&mats_full[m]);
            }
            if (lane == 0) {
                fence_proxy_async_smem();  // the stage's earlier reads before the copies
                mbar_arrive_expect_tx(&full[slot],
                                      (uint32_t)fast_stage_bytes(D) + ctl.stall_tx_bytes);
                fast_stage_rows(maps.m, a, st, smem + L.ring + slot * fast_stage_bytes(D),
                                &full[slot]);
            }
            __syncwarp();
            st.next(a, tiles_n, ntiles);
        }
        for (; ok && reduced < nsteps; ++reduced) {  // the last steps' key sums
            ok = fast_reduce_sums(a, rd, reduced, part, sums_full, sums_empty, C, lane,
                                  ctl.wait_limit_ns, abort_flag);
            rd.next(a, tiles_n, ntiles);
        }
        if (lane == 0 && (!ok || *abort_flag)) {
            // Stages the compute warps may not have waited for: wait (bounded)
            // for the copies issued into them, so none is in flight at exit.
            for (int64_t j = s > STAGES ? s - STAGES : 0; j < s; ++j)
                mbar_wait_bounded(&full[j % STAGES], (uint32_t)((j / STAGES) & 1),
                                  ctl.wait_limit_ns);
        }
    } else {
        // ------------------------------ compute warps ------------------------------
        const int i = lane, c = warp;  // tokens i and i + 32 of the tile, chunk
        const int pitch = fast_row_pitch(D);
        const int64_t row_bytes = N * 2;
        FastStep st{};
        st.locate(a, tiles_n, ntiles);
        float2 cj[4], sj[4];
        for (int64_t s = 0; s < nsteps; ++s) {
            const int slot = (int)(s % STAGES);
            const int m = (int)(st.ti & 1);
            if (st.h == 0) {
                // this tile's cos/sin for the thread's pair and chunk, for all heads
                const int half = D / 2;
                const int64_t r0 = (st.n0 + i) * half + 4 * c;
                const int64_t r1 = r0 + (int64_t)kPairs * half;
                const bool ok0 = i < st.tv, ok1 = i + kPairs < st.tv;
                const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
                const float4 c0 = ok0 ? __ldg(reinterpret_cast<const float4*>(a.rope_cos + r0)) : z;
                const float4 c1 = ok1 ? __ldg(reinterpret_cast<const float4*>(a.rope_cos + r1)) : z;
                const float4 s0 = ok0 ? __ldg(reinterpret_cast<const float4*>(a.rope_sin + r0)) : z;
                const float4 s1 = ok1 ? __ldg(reinterpret_cast<const float4*>(a.rope_sin + r1)) : z;
                cj[0] = make_float2(c0.x, c1.x); cj[1] = make_float2(c0.y, c1.y);
                cj[2] = make_float2(c0.z, c1.z); cj[3] = make_float2(c0.w, c1.w);
                sj[0] = make_float2(s0.x, s1.x); sj[1] = make_float2(s0.y, s1.y);
                sj[2] = make_float2(s0.z, s1.z); sj[3] = make_float2(s0.w, s1.w);
                ok = mbar_wait_abortable(&mats_full[m], (uint32_t)((st.ti / 2) & 1),
                                         ctl.wait_limit_ns, abort_flag);
                if (STAGED) ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            ok = mbar_wait_abortable(&full[slot], (uint32_t)((s / STAGES) & 1), ctl.wait_limit_ns,
                                     abort_flag);
            if (STAGED) ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const unsigned char* in = smem + L.ring + slot * fast_stage_bytes(D);
            const float* mats = mats_base + m * 2 * kPairs * kMatStride;
            const int64_t head_row0 = (st.b * H + st.h) * (int64_t)D + 8 * c;  // first output row
            const int64_t col = st.n0 * 2;
            float2 si = make_float2(0.f, 0.f), so = si;
            const bool va = i < st.tv, vb = i + kPairs < st.tv;
            unsigned char* ob = smem + L.out + c * 8 * kTile * 2;
            if (va || STAGED) {  // staged: the whole warp (rows past the tile end are zeros)
                fast_tensor<H16, 0, STAGED>(in, mats, cj, sj, pitch, i, c, a.k_scale,
                                            a.q_out + head_row0 * row_bytes + col, row_bytes, va,
                                            vb, si, so, ob, st.tv);
                fast_tensor<H16, 1, STAGED>(in, mats, cj, sj, pitch, i, c, a.k_scale,
                                            a.k_out + head_row0 * row_bytes + col, row_bytes, va,
                                            vb, si, so, ob, st.tv);
                fast_tensor<H16, 2, STAGED>(in, mats, cj, sj, pitch, i, c, a.k_scale,
                                            a.v_out + head_row0 * row_bytes + col, row_bytes, va,
                                            vb, si, so, ob, st.tv);
            }
            mbar_arrive(&empty[slot]);  // the stage is read
            if (st.h == H - 1) mbar_arrive(&mats_empty[m]);
            if (s >= 2) {  // the copy warp has read step s - 2's key sums
                ok = mbar_wait_abortable(&sums_empty[s & 1], (uint32_t)((s / 2 - 1) & 1),
                                         ctl.wait_limit_ns, abort_flag);
                if (STAGED) ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            float2* pc = part + (s & 1) * C * kTile + c * kTile;
            pc[i] = make_float2(si.x, so.x);
            pc[i + kPairs] = make_float2(si.y, so.y);
            mbar_arrive(&sums_full[s & 1]);
            st.next(a, tiles_n, ntiles);
        }
    }
    if (!ok) {
        *abort_flag = 1u;
        if (lane == 0) atomicOr(&g_ucpe_status, 1u);
    }
}

// ---------------------------------------------------------------------------
// Barrier-synchronised pipelined kernel: head_dim 64 or less, and 128 (where
// it measured faster than the warp-specialised kernel above), num_tokens
// even (whole token pairs, 4-byte aligned output rows), at least two heads.
//
// Work unit: a tile of 64 tokens of one batch element, all heads in turn.
// Lane i of every warp owns the token pair (2i, 2i+1); warp w owns the
// 8-channel chunk w. For each head:
//   - its Q, K, V rows (64 tokens x D, three tensors) arrive by 16-byte
//     cp.async into one stage of a ring of shared-memory stages (consecutive
//     threads copy consecutive chunks of a row), issued several heads ahead;
//   - each thread widens, projects, rotates and rounds its two tokens x eight
//     channels of each tensor with packed fp32x2 instructions and stores one
//     32-bit word (both tokens) per channel straight to [B, H, D, N];
//   - the per-chunk key sums go to shared memory and are added per token, in a
//     fixed order, one head later (so one CTA barrier per head suffices).
// Padding: a token pair's two rows take 2D*2 + 16 bytes of a stage, so that
// the 16-byte chunks that eight consecutive lanes read fall in distinct banks;
// a pair's interleaved matrices take 144 bytes for the same reason.
__host__ __device__ inline int sync_pair_stride(int D) { return 4 * D + 16; }  // bytes
__host__ __device__ inline int sync_stage_bytes(int D) { return 3 * kPairs * sync_pair_stride(D); }

struct SyncLayout {
    int ring, mats, part, total, stages;
};

// Stages: as many as fit (at most 4) beside two matrix and two key-sum buffers.
__host__ __device__ inline SyncLayout sync_layout(int D, int stages) {
    SyncLayout L;
    const int C = D / 8;
    L.stages = stages;
    L.ring = 0;
    L.mats = stages * sync_stage_bytes(D);            // [2][2][32][kMatStride] f32
    L.part = L.mats + 2 * 2 * kPairs * kMatStride * 4;  // [2][C][64] float2
    L.total = L.part + 2 * C * kTile * 8;
    return L;
}

__device__ __forceinline__ void cp_async16z(void* dst_smem, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst_smem)),
                 "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

template <int K>
__device__ __forceinline__ void cp_async_wait_pending() {
    asm volatile("cp.async.wait_group %0;" ::"n"(K) : "memory");
}


// The matrices of a tile's tokens into matrix buffer `mats`, interleaved by
// token pairs (4-byte copies; tokens past the tile's end read as zeros).
__device__ __forceinline__ void sync_stage_mats(const UcpeArgs& a, const FastStep& st, float* mats) {
    for (int f = threadIdx.x; f < kTile * 32; f += blockDim.x) {
        const int e = f & 15, m = (f >> 4) & 1, t = f >> 5;
        const bool ok = t < st.tv;
        const float* src =
            (m ? a.proj_kv : a.proj_q) + (ok ? (st.b * a.num_tokens + st.n0 + t) * 16 + e : 0);
        cp_async4(mats + (m * kPairs + (t >> 1)) * kMatStride + e * 2 + (t & 1), src, ok);
    }
}

// The warp rank that decides which token rows a warp copies. 64 rows over
// 2 * warps half-warps leave some half-warps one row more than others; the
// rotation gives the longer share to warps 4.. and keeps it off warps 0 and 1,
// which also add up the key sums, so that no warp is late at the barrier.
__device__ __forceinline__ int sync_copy_rank(int warp, int nwarps) {
    return nwarps > 4 ? (warp + nwarps - 4) % nwarps : warp;
}

// One head's Q, K, V rows of a tile into ring stage `buf` (16-byte copies;
// sixteen lanes per token row, lane k copying chunk k of that token's Q, K and
// V rows; a lane takes tokens t0, t0 + 2 * warps, ... with t0 from its warp's
// copy rank; tokens past the tile's end read as zeros). `off` is the byte offset of chunk k of token t0's row at
// head 0 of the tile (sync_row_offset); successive tokens of the lane are
// 2 * warps rows apart.
__device__ __forceinline__ void sync_stage_head(const UcpeArgs& a, const FastStep& st, int64_t off,
                                                unsigned char* buf) {
    const int D = a.head_dim, C = D / 8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int ps = sync_pair_stride(D);
    const int k4 = lane & 15;
    if (k4 >= C) return;
    const int64_t step = (int64_t)2 * nwarps * a.heads * D * 2;
    int64_t o = off + (int64_t)st.h * D * 2;
    for (int t = 2 * sync_copy_rank(warp, nwarps) + (lane >> 4); t < kTile; t += 2 * nwarps, o += step) {
        const bool ok = t < st.tv;
        const int64_t src = ok ? o : 0;
        unsigned char* dst = buf + (t >> 1) * ps + (t & 1) * 2 * D + 16 * k4;
        cp_async16z(dst, a.q + src, ok);
        cp_async16z(dst + kPairs * ps, a.k + src, ok);
        cp_async16z(dst + 2 * kPairs * ps, a.v + src, ok);
    }
}

// Byte offset (from the tensor base) of chunk k4 of this lane's first token
// row at head 0 of the tile.
__device__ __forceinline__ int64_t sync_row_offset(const UcpeArgs& a, const FastStep& st) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int t0 = 2 * sync_copy_rank(warp, nwarps) + (lane >> 4);
    return ((st.b * a.num_tokens + st.n0 + t0) * a.heads * a.head_dim + 8 * (lane & 15)) * 2;
}

// Issue the copies of step `st` into ring stage `slot` (its head's rows; at a
// tile's first head also the tile's matrices) and commit them as one group,
// empty if the step is past the end.
__device__ __forceinline__ void sync_issue(const UcpeArgs& a, const FastStep& st, int64_t off,
                                           int slot,
                                           unsigned char* smem, const SyncLayout& L) {
    if (st.valid) {
        sync_stage_head(a, st, off, smem + L.ring + slot * sync_stage_bytes(a.head_dim));
        if (st.h == 0)
            sync_stage_mats(a, st, reinterpret_cast<float*>(smem + L.mats) +
                                       (st.ti & 1) * 2 * kPairs * kMatStride);
    }
    cp_async_commit();
}

// Tensor X of this thread's token pair and chunk: widen, ReLU (Q, K), project,
// rotate (Q, K), scale (K), round; one packed word per channel stored straight
// to the output. For K, the pair's sums of squares go to si/so.
template <bool H16, int X>
__device__ __forceinline__ void sync_tensor(const unsigned char* in, const float* mats,
                                            const float2 (&cj)[4], const float2 (&sj)[4],
                                            int D, int pp, int c, float k_scale, uint8_t* out_row0,
                                            int64_t row_bytes, float2& si, float2& so) {
    const int ps = sync_pair_stride(D);
    const uint4 ra = *reinterpret_cast<const uint4*>(in + (X * kPairs + pp) * ps + 16 * c);
    const uint4 rb = *reinterpret_cast<const uint4*>(in + (X * kPairs + pp) * ps + 2 * D + 16 * c);
    uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
    uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
    if (X < 2) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            wa[e] = relu2<H16>(wa[e]);
            wb[e] = relu2<H16>(wb[e]);
        }
    }
    float2 x[8], y[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) widen_pair<H16>(wa[e], wb[e], x[2 * e], x[2 * e + 1]);
    const float* m = mats + ((X == 0 ? 0 : kPairs) + pp) * kMatStride;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 r01 = *reinterpret_cast<const float4*>(m + 8 * i);
        const float4 r23 = *reinterpret_cast<const float4*>(m + 8 * i + 4);
        const float2 m0 = make_float2(r01.x, r01.y), m1 = make_float2(r01.z, r01.w);
        const float2 m2 = make_float2(r23.x, r23.y), m3 = make_float2(r23.z, r23.w);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            const float2* xb = x + 4 * blk;
            y[4 * blk + i] = fma2(m3, xb[3], fma2(m2, xb[2], fma2(m1, xb[1], mul2(m0, xb[0]))));
        }
    }
    if (X == 1) {
        float2 a2 = make_float2(0.f, 0.f), b2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            a2 = fma2(x[e], x[e], a2);
            b2 = fma2(y[e], y[e], b2);
        }
        si = a2;
        so = b2;
    }
    if (X < 2) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 ya = y[2 * j], yb = y[2 * j + 1];
            const float2 bs = mul2(yb, sj[j]);
            y[2 * j] = fma2(ya, cj[j], make_float2(-bs.x, -bs.y));
            y[2 * j + 1] = fma2(yb, cj[j], mul2(ya, sj[j]));
        }
    }
    if (X == 1) {
        const float2 ks = make_float2(k_scale, k_scale);
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = mul2(y[e], ks);
    }
    uint8_t* o = out_row0 + 4 * pp;
#pragma unroll
    for (int e = 0; e < 8; ++e)
        *reinterpret_cast<uint32_t*>(o + (int64_t)e * row_bytes) = f2_to_act2<H16>(y[e]);
}

template <bool H16, int STAGES>
__global__ void __launch_bounds__(512, 1) ucpe_sync_kernel(const UcpeArgs a) {
    const int D = a.head_dim, C = D / 8, H = a.heads;
    const int64_t N = a.num_tokens;
    const int64_t tiles_n = (N + kTile - 1) / kTile;
    const int64_t ntiles = a.batch * tiles_n;
    const int tid = threadIdx.x;
    const int pp = tid & 31, c = tid >> 5;  // token pair, chunk
    const bool key_scaled = a.k_scale != 0.0f;
    const SyncLayout L = sync_layout(D, STAGES);

    extern __shared__ __align__(128) unsigned char smem[];
    float2* part = reinterpret_cast<float2*>(smem + L.part);  // [2][C][64]

    if ((int64_t)blockIdx.x >= ntiles) return;
    // this CTA's steps: its tiles x heads
    const int64_t my_tiles = (ntiles - 1 - blockIdx.x) / gridDim.x + 1;
    const int64_t nsteps = my_tiles * H;
    const int64_t row_bytes = N * 2;

    griddep_wait();
    griddep_launch_dependents();

    FastStep st{}, ahead{};
    st.locate(a, tiles_n, ntiles);
    ahead = st;
    int64_t off = sync_row_offset(a, ahead);  // of the tile `ahead` is in
    for (int k = 0; k < STAGES - 1; ++k) {
        sync_issue(a, ahead, off, k, smem, L);
        ahead.next(a, tiles_n, ntiles);
        if (ahead.h == 0) off = sync_row_offset(a, ahead);
    }

    float2 cj[4], sj[4];
    FastStep prev{};
    for (int64_t s = 0; s < nsteps; ++s) {
        // At a tile's first head its cos/sin go out first: they do not depend
        // on shared memory, so their latency overlaps the wait and the barrier.
        if (st.h == 0) {
            // this tile's cos/sin for the thread's pair and chunk, for all heads
            const int half = D / 2;
            const int64_t r0 = (st.n0 + 2 * pp) * half + 4 * c;
            const bool ok0 = 2 * pp < st.tv, ok1 = 2 * pp + 1 < st.tv;
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 c0 = ok0 ? __ldg(reinterpret_cast<const float4*>(a.rope_cos + r0)) : z;
            const float4 c1 = ok1 ? __ldg(reinterpret_cast<const float4*>(a.rope_cos + r0 + half)) : z;
            const float4 s0 = ok0 ? __ldg(reinterpret_cast<const float4*>(a.rope_sin + r0)) : z;
            const float4 s1 = ok1 ? __ldg(reinterpret_cast<const float4*>(a.rope_sin + r0 + half)) : z;
            cj[0] = make_float2(c0.x, c1.x); cj[1] = make_float2(c0.y, c1.y);
            cj[2] = make_float2(c0.z, c1.z); cj[3] = make_float2(c0.w, c1.w);
            sj[0] = make_float2(s0.x, s1.x); sj[1] = make_float2(s0.y, s1.y);
            sj[2] = make_float2(s0.z, s1.z); sj[3] = make_float2(s0.w, s1.w);
        }
        cp_async_wait_pending<STAGES - 2>();  // this step's group is complete
        __syncthreads();
        // The stage of step s - 1 is free now: refill it with step s + STAGES - 1.
        sync_issue(a, ahead, off, (int)((s + STAGES - 1) % STAGES), smem, L);
        ahead.next(a, tiles_n, ntiles);
        if (ahead.h == 0) off = sync_row_offset(a, ahead);

        // Key sums of the previous step (written before the barrier above).
        if (s > 0 && a.inflation_sq) {
            const float2* pprev = part + ((s - 1) & 1) * C * kTile;
            for (int t = tid; t < prev.tv; t += blockDim.x) {
                float s_in = 0.f, s_out = 0.f;
                for (int cc = 0; cc < C; ++cc) {
                    const float2 v = pprev[cc * kTile + t];
                    s_in += v.x;
                    s_out += v.y;
                }
                a.inflation_sq[(prev.b * H + prev.h) * N + prev.n0 + t] =
                    (s_in > 0.f && key_scaled) ? s_out / s_in : 1.0f;
            }
        }

        const int64_t ti = st.ti;
        const unsigned char* in = smem + L.ring + (int)(s % STAGES) * sync_stage_bytes(D);
        const float* mats = reinterpret_cast<const float*>(smem + L.mats) + (ti & 1) * 2 * kPairs * kMatStride;
        const int64_t head_row0 = (st.b * H + st.h) * (int64_t)D + 8 * c;  // first output row
        const int64_t col = st.n0 * 2;
        float2 si = make_float2(0.f, 0.f), so = si;
        if (2 * pp < st.tv) {
            sync_tensor<H16, 0>(in, mats, cj, sj, D, pp, c, a.k_scale,
                                a.q_out + head_row0 * row_bytes + col, row_bytes, si, so);
            sync_tensor<H16, 1>(in, mats, cj, sj, D, pp, c, a.k_scale,
                                a.k_out + head_row0 * row_bytes + col, row_bytes, si, so);
            sync_tensor<H16, 2>(in, mats, cj, sj, D, pp, c, a.k_scale,
                                a.v_out + head_row0 * row_bytes + col, row_bytes, si, so);
        }
        *reinterpret_cast<float4*>(part + (s & 1) * C * kTile + c * kTile + 2 * pp) =
            make_float4(si.x, so.x, si.y, so.y);
        prev = st;
        st.next(a, tiles_n, ntiles);
    }
    // The last step's key sums.
    __syncthreads();
    if (nsteps > 0 && a.inflation_sq) {
        const float2* pprev = part + ((nsteps - 1) & 1) * C * kTile;
        for (int t = tid; t < prev.tv; t += blockDim.x) {
            float s_in = 0.f, s_out = 0.f;
            for (int cc = 0; cc < C; ++cc) {
                const float2 v = pprev[cc * kTile + t];
                s_in += v.x;
                s_out += v.y;
            }
            a.inflation_sq[(prev.b * H + prev.h) * N + prev.n0 + t] =
                (s_in > 0.f && key_scaled) ? s_out / s_in : 1.0f;
        }
    }
    cp_async_wait_all();
}

template <typename K, typename... Args>
cudaError_t launch_pdl(K kern, int grid, int block, int smem, cudaStream_t stream,
                       const Args&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled, looked up once through the runtime (no link
// against the driver library); null if the driver does not offer it.
EncodeTiled encode_tiled() {
    static std::once_flag once;
    static EncodeTiled fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// The three row maps of a camera-prep call; false if one cannot be encoded.
bool encode_maps(const UcpeArgs& a, UcpeMaps* maps) {
    const EncodeTiled enc = encode_tiled();
    if (!enc) return false;
    const int D = a.head_dim;
    const cuuint64_t dims[2] = {(cuuint64_t)a.heads * D, (cuuint64_t)(a.batch * a.num_tokens)};
    const cuuint64_t strides[1] = {(cuuint64_t)a.heads * D * 2};
    const cuuint32_t box[2] = {(cuuint32_t)fast_row_elems(D), (cuuint32_t)kTile};
    const cuuint32_t estr[2] = {1, 1};
    const uint8_t* base[3] = {a.q, a.k, a.v};
    for (int X = 0; X < 3; ++X) {
        if (enc(&maps->m[X], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                const_cast<void*>(static_cast<const void*>(base[X])), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    return true;
}

}  // namespace

cudaError_t launch_fast(const UcpeArgs& a, const UcpeControl& ctl, cudaStream_t stream,
                        LaunchInfo* info, bool* used) {
    *used = false;
    const int D = a.head_dim;
    const int block = 32 * (D / 8 + 1);  // D/8 compute warps and the copy warp
    // The row maps address rows with 32-bit coordinates and take whole
    // 64-row boxes; a row of the box takes fast_row_elems(D) <= 2D columns.
    const int64_t rows = a.batch * a.num_tokens;
    if (!ctl.device_inputs || a.heads < 2 || rows < kTile || rows > INT32_MAX) return cudaSuccess;
    UcpeMaps maps;
    if (!encode_maps(a, &maps)) return cudaSuccess;  // the general kernel runs instead
    int sms = 0, optin = 0, dev = 0;
    cudaError_t e = cached_sm_count(&sms);
    if (e != cudaSuccess) return e;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    // A tile's matrices are double-buffered and the copy warp writes a tile's
    // only after the compute warps are done with the tile two before it, so
    // the ring may run at most heads + 1 steps ahead. Of the ring depths that
    // fit, take the one that keeps the most head stages in flight per SM
    // (CTAs per SM x (depth - 1)), the deeper ring on a tie.
    int stages = 0, per_sm = 0, best = 0;
    bool staged = false;
    void (*kern)(const UcpeArgs, const UcpeMaps, const UcpeControl) = nullptr;
    for (int s = std::min(4, a.heads + 1); s >= 3; --s) {
        // Rows staged through shared memory and written with 16-byte stores
        // when num_tokens is 8 mod 16: its rows then start 16 bytes past a
        // 32-byte sector, where the direct 16-bit stores touch three sectors
        // per 64-byte half row (117 -> 106.5 us at head_dim 112, 20 heads);
        // elsewhere the extra instructions cost more than they save.
        for (int sg = (a.num_tokens % 16 == 8) ? 1 : 0; sg >= 0; --sg) {
            if (fast_layout(D, s, sg).total > optin) continue;
            void (*k)(const UcpeArgs, const UcpeMaps, const UcpeControl) =
                sg ? (s == 4 ? (a.act_f16 ? ucpe_fast_kernel<true, 4, true>
                                          : ucpe_fast_kernel<false, 4, true>)
                             : (a.act_f16 ? ucpe_fast_kernel<true, 3, true>
                                          : ucpe_fast_kernel<false, 3, true>))
                   : (s == 4 ? (a.act_f16 ? ucpe_fast_kernel<true, 4, false>
                                          : ucpe_fast_kernel<false, 4, false>)
                             : (a.act_f16 ? ucpe_fast_kernel<true, 3, false>
                                          : ucpe_fast_kernel<false, 3, false>));
            int n = 0;
            if (cached_smem_and_occupancy(reinterpret_cast<const void*>(k), block,
                                          fast_layout(D, s, sg).total, &n) != cudaSuccess) {
                cudaGetLastError();
                continue;
            }
            if (n * (s - 1) > best) {
                best = n * (s - 1);
                stages = s;
                staged = sg;
                per_sm = n;
                kern = k;
            }
        }
    }
    if (!kern) return cudaSuccess;  // does not fit: the general kernel runs instead
    const FastLayout L = fast_layout(D, stages, staged);
    const int64_t tiles = a.batch * ((a.num_tokens + kTile - 1) / kTile);
    const int grid = (int)std::min<int64_t>((int64_t)sms * per_sm, tiles);
    e = launch_pdl(kern, grid, block, L.total, stream, a, maps, ctl);
    if (e != cudaSuccess) {
        cudaGetLastError();
        forget_kernel(reinterpret_cast<const void*>(kern));
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block, L.total, &per_sm);
        if (e == cudaSuccess) e = launch_pdl(kern, grid, block, L.total, stream, a, maps, ctl);
    }
    *used = true;
    if (info) {
        info->grid = grid;
        info->block = block;
        info->smem = L.total;
        info->kernel_id = 5100 + 10 * stages + (a.act_f16 ? 1 : 0) + (staged ? 200 : 0);
    }
    return e;
}

cudaError_t launch_sync(const UcpeArgs& a, cudaStream_t stream, LaunchInfo* info, bool* used) {
    *used = false;
    const int D = a.head_dim;
    const int block = 4 * D;  // 32 token pairs x D/8 chunks
    int sms = 0, optin = 0, dev = 0;
    cudaError_t e = cached_sm_count(&sms);
    if (e != cudaSuccess) return e;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    // A tile's matrices are double-buffered, so the ring may run at most
    // heads + 1 steps ahead (the next-but-one tile's matrices must not land
    // while a tile still reads its own). Of the ring depths that fit, take the
    // one that keeps the most head stages in flight per SM (CTAs per SM x
    // (depth - 1)), the deeper ring on a tie.
    int stages = 0, per_sm = 0, best = 0;
    void (*kern)(const UcpeArgs) = nullptr;
    for (int s = std::min(4, a.heads + 1); s >= 3; --s) {
        if (sync_layout(D, s).total > optin) continue;
        void (*k)(const UcpeArgs) =
            s == 4 ? (a.act_f16 ? ucpe_sync_kernel<true, 4> : ucpe_sync_kernel<false, 4>)
                   : (a.act_f16 ? ucpe_sync_kernel<true, 3> : ucpe_sync_kernel<false, 3>);
        int n = 0;
        if (cached_smem_and_occupancy(reinterpret_cast<const void*>(k), block,
                                      sync_layout(D, s).total, &n) != cudaSuccess) {
            cudaGetLastError();
            continue;
        }
        if (n * (s - 1) > best) {
            best = n * (s - 1);
            stages = s;
            per_sm = n;
            kern = k;
        }
    }
    if (!kern) return cudaSuccess;  // does not fit: the general kernel runs instead
    const SyncLayout L = sync_layout(D, stages);
    const int64_t tiles = a.batch * ((a.num_tokens + kTile - 1) / kTile);
    const int grid = (int)std::min<int64_t>((int64_t)sms * per_sm, tiles);
    e = launch_pdl(kern, grid, block, L.total, stream, a);
    if (e != cudaSuccess) {
        cudaGetLastError();
        forget_kernel(reinterpret_cast<const void*>(kern));
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block, L.total, &per_sm);
        if (e == cudaSuccess) e = launch_pdl(kern, grid, block, L.total, stream, a);
    }
    *used = true;
    if (info) {
        info->grid = grid;
        info->block = block;
        info->smem = L.total;
        info->kernel_id = 5200 + 10 * stages + (a.act_f16 ? 1 : 0);
    }
    return e;
}

cudaError_t read_ucpe_status(uint32_t* out, int clear, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_ucpe_status, sizeof(uint32_t), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && clear) {
        const uint32_t zero = 0;
        e = cudaMemcpyToSymbolAsync(g_ucpe_status, &zero, sizeof(uint32_t), 0,
                                    cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    }
    return e;
}

cudaError_t launch_ucpe(const UcpeArgs& a, const UcpeControl& ctl, cudaStream_t stream,
                        LaunchInfo* info) {
    const int D = a.head_dim;
    if (D < 8 || D > 256 || D % 8 != 0) return cudaErrorInvalidValue;
    // The warp-specialised kernel for head_dim 72..120, the barrier-
    // synchronised one (even token counts) for the other head_dims up to 128
    // and where the first cannot run; the general kernel for the rest.
    if (D <= kFastMaxD) {
        bool used = false;
        cudaError_t e = cudaSuccess;
        if (D > 64 && D <= kWsMaxD) {
            e = launch_fast(a, ctl, stream, info, &used);
            if (used || e != cudaSuccess) return e;
        }
        if (a.num_tokens % 2 == 0) {
            e = launch_sync(a, stream, info, &used);
            if (used || e != cudaSuccess) return e;
        }
    }
    const int block = ucpe_block(D), smem = ucpe_smem(D);
    void (*kern)(const UcpeArgs) =
        a.act_f16 ? ucpe_prep_kernel<true, false> : ucpe_prep_kernel<false, false>;
    int sms = 0, per_sm = 0;
    cudaError_t e = cached_sm_count(&sms);
    if (e != cudaSuccess) return e;
    e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block, smem, &per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    // Whole tiles per CTA (the tile's matrices and cos/sin rows staged once
    // for all its heads) unless that leaves the last round of tiles so uneven
    // that it takes over a quarter more (tile, head) rounds than single units.
    const int64_t slots = (int64_t)sms * per_sm;
    const int64_t tiles_bt = a.batch * ((a.num_tokens + kTile - 1) / kTile);
    const int64_t rounds_tile = (tiles_bt + slots - 1) / slots * a.heads;
    const int64_t rounds_unit = (tiles_bt * a.heads + slots - 1) / slots;
    const bool tile_major = a.heads > 1 && 4 * rounds_tile <= 5 * rounds_unit;
    if (tile_major) {
        kern = a.act_f16 ? ucpe_prep_kernel<true, true> : ucpe_prep_kernel<false, true>;
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block, smem, &per_sm);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
    }
    const int64_t tiles = tiles_bt * (tile_major ? 1 : a.heads);
    const int grid = (int)std::min<int64_t>((int64_t)sms * per_sm, tiles);
    e = launch_pdl(kern, grid, block, smem, stream, a);
    if (e != cudaSuccess) {
        cudaGetLastError();
        forget_kernel(reinterpret_cast<const void*>(kern));
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block, smem, &per_sm);
        if (e == cudaSuccess) e = launch_pdl(kern, grid, block, smem, stream, a);
    }
    if (info) {
        info->grid = grid;
        info->block = block;
        info->smem = smem;
        info->kernel_id = 5000 + (a.act_f16 ? 1 : 0) + (tile_major ? 2 : 0);
    }
    return e;
}

}  // namespace qknr
