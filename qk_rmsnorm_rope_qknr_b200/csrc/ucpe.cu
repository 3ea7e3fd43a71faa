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
// The work is a stream over HBM (about 1.5 flops per byte), so the kernel is
// built for coalescing on both sides of the transpose:
//   - work unit: a tile of 64 consecutive tokens of one (batch, head), tiles
//     numbered with the head fastest, so that the tiles in flight at once
//     share their tokens' cos/sin rows and matrices in L2;
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
// The 4x4 matrices of the tile's tokens are staged in shared memory once per
// tile; the per-chunk key sums are summed per token in a fixed order, so the
// results do not depend on the launch shape.
#include "common.cuh"
#include "launch.h"
#include "launch_cache.h"

#include <algorithm>

namespace qknr {
namespace {

constexpr int kTile = 64;        // tokens per tile (one 128-byte output row)
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
    if (X == 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] *= k_scale;
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

template <bool H16>
__global__ void __launch_bounds__(512) ucpe_prep_kernel(const UcpeArgs a) {
    const int D = a.head_dim, C = D / 8, H = a.heads;
    const int64_t N = a.num_tokens;
    const int64_t tiles_n = (N + kTile - 1) / kTile;
    const int64_t ntiles = a.batch * tiles_n * H;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const bool vec_out = (N & 7) == 0;

    extern __shared__ __align__(16) unsigned char smem[];
    unsigned char* stage = smem;  // [3][D][kTile] 16-bit, swizzled rows
    float* proj = reinterpret_cast<float*>(smem + 3 * D * kTile * 2);  // [kTile][kProjStride]
    float* cosr = proj + kTile * kProjStride;                            // [kTile][D/2]
    float* sinr = cosr + kTile * (D / 2);                                // [kTile][D/2]
    float2* part = reinterpret_cast<float2*>(sinr + kTile * (D / 2));   // [kTile][C]

    // This thread's item: tokens 4p..4p+3 of the tile, channels 8c..8c+7.
    const int p = tid / C, c = tid - (tid / C) * C;
    const bool has_item = tid < (kTile / 4) * C;

    int64_t tile = blockIdx.x;
    if (tile >= ntiles) return;
    const int64_t step_bt = (int64_t)gridDim.x / H;
    const int step_h = (int)((int64_t)gridDim.x - step_bt * H);
    TileCursor cur;
    cur.h = (int)(tile % H);
    cur.tn = tile / H;
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

        // The next tile's inputs go out before this tile's stores.
        tile += gridDim.x;
        const bool more = tile < ntiles;
        if (more) {
            cur.advance(step_bt, step_h, H, tiles_n);
            const int64_t nn0 = cur.tn * kTile;
            const int ntv = (int)min((int64_t)kTile, N - nn0);
            stage_token_inputs(a, cur.b, nn0, ntv, tid, nthr, proj, cosr, sinr);
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
                a.inflation_sq[(b * H + h) * N + n0 + t] = si > 0.f ? so / si : 1.0f;
            }
        }
        if (!more) break;
        cp_async_wait_all();
        __syncthreads();
    }
}

template <typename K>
cudaError_t launch_pdl(K kern, int grid, int block, int smem, cudaStream_t stream,
                       const UcpeArgs& args) {
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
    return cudaLaunchKernelEx(&cfg, kern, args);
}

}  // namespace

cudaError_t launch_ucpe(const UcpeArgs& a, cudaStream_t stream, LaunchInfo* info) {
    const int D = a.head_dim;
    if (D < 8 || D > 256 || D % 8 != 0) return cudaErrorInvalidValue;
    const int block = ucpe_block(D), smem = ucpe_smem(D);
    void (*kern)(const UcpeArgs) = a.act_f16 ? ucpe_prep_kernel<true> : ucpe_prep_kernel<false>;
    int sms = 0, per_sm = 0;
    cudaError_t e = cached_sm_count(&sms);
    if (e != cudaSuccess) return e;
    e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block, smem, &per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t tiles = a.batch * ((a.num_tokens + kTile - 1) / kTile) * a.heads;
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
        info->kernel_id = 5000 + (a.act_f16 ? 1 : 0);
    }
    return e;
}

}  // namespace qknr
