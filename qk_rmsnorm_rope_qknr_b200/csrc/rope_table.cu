// Table-driven per-head Q/K RMSNorm + RoPE.
//
// Computes the operation of "vllm_omni.diffusion.layers.fused_qk_norm_rope"
// (vLLM-Omni API docs; contract bullets and fused_qk_norm_rope): each head of
// q [T, Hq, D] and k [T, Hk, D] is RMS-normalised over its D channels, scaled
// by a [D] weight and rotated by the token's row of a [T, rotary_dim] cos/sin
// table, pairs (2j, 2j+1) (interleaved) or (j, j + rotary_dim/2) (half split);
// channels >= rotary_dim are normalised only. Activations (and weights, and a
// 16-bit table) are bf16 or IEEE binary16; the arithmetic is fp32 either way.
//
// Fast kernel: a head is a group of GS lanes (GS = next power of two of D/16);
// lane l of the group owns two 16-byte vectors of the head, chosen so that
// every rotation pair sits inside the lane: half split -> vectors l and
// l + rotary_dim/16 for l < rotary_dim/16, the pass-through vectors two by two
// after that; interleaved -> vectors l and l + D/16. The group's sum of
// squares is a GS-lane shuffle reduction: no barrier. A warp item is 4 rounds
// of 32/GS heads of one token. Each warp keeps a ring of shared-memory buffers
// that its lane 0 fills with bulk asynchronous copies (the item's q heads, k
// heads and the token's table row) a ring ahead of use; the lane's cos/sin for
// the token (the same for every head) are read once per item. Which of a
// lane's two vectors each shared load fetches is planned on the host so that
// no two lanes of a load phase share a bank group (LaneMap); the norm weights
// sit in shared memory as fp32 in the matching lane-major order.
//
// General kernel: one warp per head through shared memory, for the shapes and
// alignments the fast kernel does not take.
#include "common.cuh"
#include "launch.h"
#include "launch_cache.h"

#include <algorithm>
#include <mutex>
#include <unordered_map>

namespace qknr {

__device__ unsigned int g_table_status;

namespace {

constexpr int kBlock = 256;
constexpr int kUnroll = 4;

// The same reads from a table row staged in shared memory (plain loads: the
// read-only global path must not see a shared address). A 16-bit table has the
// activation type.
template <bool F32, bool H16>
__device__ __forceinline__ void smem_cos_sin8(const uint8_t* row, int col, int half,
                                              float (&c)[8], float (&s)[8]) {
    if constexpr (F32) {
        const float4* pc = reinterpret_cast<const float4*>(row + (size_t)col * 4);
        const float4* ps = reinterpret_cast<const float4*>(row + (size_t)(half + col) * 4);
        const float4 c0 = pc[0], c1 = pc[1], s0 = ps[0], s1 = ps[1];
        c[0] = c0.x; c[1] = c0.y; c[2] = c0.z; c[3] = c0.w;
        c[4] = c1.x; c[5] = c1.y; c[6] = c1.z; c[7] = c1.w;
        s[0] = s0.x; s[1] = s0.y; s[2] = s0.z; s[3] = s0.w;
        s[4] = s1.x; s[5] = s1.y; s[6] = s1.z; s[7] = s1.w;
    } else {
        const uint4 cv = *reinterpret_cast<const uint4*>(row + (size_t)col * 2);
        const uint4 sv = *reinterpret_cast<const uint4*>(row + (size_t)(half + col) * 2);
        const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w}, sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float2 c2 = act2_to_f2<H16>(cw[m]), s2 = act2_to_f2<H16>(sw[m]);
            c[2 * m] = c2.x; c[2 * m + 1] = c2.y;
            s[2 * m] = s2.x; s[2 * m + 1] = s2.y;
        }
    }
}

template <bool F32, bool H16>
__device__ __forceinline__ void smem_cos_sin4(const uint8_t* row, int col, int half, float* c,
                                              float* s) {
    if constexpr (F32) {
        const float4 cv = *reinterpret_cast<const float4*>(row + (size_t)col * 4);
        const float4 sv = *reinterpret_cast<const float4*>(row + (size_t)(half + col) * 4);
        c[0] = cv.x; c[1] = cv.y; c[2] = cv.z; c[3] = cv.w;
        s[0] = sv.x; s[1] = sv.y; s[2] = sv.z; s[3] = sv.w;
    } else {
        const uint2 cv = *reinterpret_cast<const uint2*>(row + (size_t)col * 2);
        const uint2 sv = *reinterpret_cast<const uint2*>(row + (size_t)(half + col) * 2);
        const float2 c0 = act2_to_f2<H16>(cv.x), c1 = act2_to_f2<H16>(cv.y);
        const float2 s0 = act2_to_f2<H16>(sv.x), s1 = act2_to_f2<H16>(sv.y);
        c[0] = c0.x; c[1] = c0.y; c[2] = c1.x; c[3] = c1.y;
        s[0] = s0.x; s[1] = s0.y; s[2] = s1.x; s[3] = s1.y;
    }
}

// Bytes of one ring buffer: the item's heads, then the token's table row.
__host__ __device__ inline int table_stage_bytes(int per_item, int D, int R, int tb) {
    return (per_item * D * 2 + R * tb + 15) & ~15;
}

// Per-lane plan of the fast kernel, chosen on the host (make_lane_map): the
// two 16-byte vectors of its head that a lane holds, which of them its first
// and its second shared-memory load fetch, and how they rotate. The order is
// picked so that the 8 lanes of each 128-bit load phase hit 8 different bank
// groups. For a half-split pair whose loads are swapped the lane negates its
// sines, which keeps one rotation formula for both orders.
struct LaneMap {
    uint32_t lane[32];
};
constexpr uint32_t kLmFirst = 0x1Fu;          // bits 0-4: vector of the first load
constexpr int kLmSecondShift = 5;             // bits 5-9: vector of the second load
constexpr uint32_t kLmSwapped = 1u << 10;     // half-split pair loaded (b, a)
constexpr uint32_t kLmAcross = 1u << 11;      // the two vectors pair up (half split)
constexpr uint32_t kLmRot1 = 1u << 12;        // first vector's adjacent pairs rotate
constexpr uint32_t kLmRot2 = 1u << 13;        // second vector's adjacent pairs rotate
constexpr uint32_t kLmActive = 1u << 14;      // the lane holds part of a head
constexpr int kWsmBytes = 2 * 4 * 32 * 16;    // weights: [q|k][4 quarter-vectors][32 lanes] float4

template <int GS, bool IL, bool F32, bool H16>
__global__ void __launch_bounds__(kBlock)
    rope_table_bulk(const RopeTableArgs a, const __grid_constant__ LaneMap m) {
    constexpr int HR = 32 / GS;  // heads per warp round
    const int D = a.head_dim, R = a.rotary_dim;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane / GS;
    const uint32_t plan = m.lane[lane];
    const bool active = (plan & kLmActive) != 0;
    const int v1 = (int)(plan & kLmFirst), v2 = (int)((plan >> kLmSecondShift) & kLmFirst);
    const bool across = (plan & kLmAcross) != 0, swapped = (plan & kLmSwapped) != 0;
    const bool rot1 = (plan & kLmRot1) != 0, rot2 = (plan & kLmRot2) != 0;
    const int H = a.hq + a.hk;
    const int per_item = kUnroll * HR;               // heads of one token per warp item
    const int cpt = (H + per_item - 1) / per_item;   // items per token
    const int64_t items = a.num_tokens * cpt;
    const int tb = F32 ? 4 : 2;  // table element bytes
    const int stages = a.stages;
    const int sbytes = table_stage_bytes(per_item, D, R, tb);

    extern __shared__ __align__(128) unsigned char smem[];
    float4* wsm = reinterpret_cast<float4*>(smem);                  // see kWsmBytes
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWsmBytes);  // [warps][stages]
    unsigned char* rings = smem + kWsmBytes + ((kBlock / 32) * stages * 8 + 127) / 128 * 128;
    uint64_t* full = bars + warp * stages;
    unsigned char* ring = rings + (size_t)warp * stages * sbytes;

    const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t n_local = warp_id < items ? (items - 1 - warp_id) / nwarps + 1 : 0;
    // item -> (token, chunk), stepped by nwarps without dividing per item
    const int64_t dt = nwarps / cpt;
    const int dchunk = (int)(nwarps - dt * cpt);

    // Issue the copies of one item into ring buffer `s` (lane 0 only).
    auto issue = [&](int64_t t, int chunk, int s) {
        const int h0 = chunk * per_item, h1 = min(h0 + per_item, H);
        const int q1 = min(h1, a.hq), k0 = max(h0, a.hq);
        const uint32_t qbytes = h0 < a.hq ? (uint32_t)(q1 - h0) * D * 2 : 0;
        const uint32_t kbytes = h1 > a.hq ? (uint32_t)(h1 - k0) * D * 2 : 0;
        unsigned char* dst = ring + (size_t)s * sbytes;
        mbar_arrive_expect_tx(&full[s], qbytes + kbytes + (uint32_t)(R * tb) + a.stall_tx_bytes);
        if (qbytes)
            bulk_load(dst, a.q + ((size_t)t * a.q_stride + (size_t)h0 * D) * 2, qbytes, &full[s]);
        if (kbytes)
            bulk_load(dst + qbytes, a.k + ((size_t)t * a.k_stride + (size_t)(k0 - a.hq) * D) * 2,
                      kbytes, &full[s]);
        bulk_load(dst + (size_t)per_item * D * 2, a.table + (size_t)t * R * tb, (uint32_t)(R * tb),
                  &full[s]);
    };

    if (lane == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    // Global memory only after the previous kernel on the stream is done (a
    // no-op unless launched as a programmatic dependent launch).
    griddep_wait();
    griddep_launch_dependents();
    // Weights as fp32, laid out per lane: entry (k, lane) of q or k holds the
    // channels 4k'..4k'+3 of the lane's vector (k < 2 ? first : second), k' =
    // k & 1, so that each of a lane's four weight loads reads 32 consecutive
    // float4 across the warp.
    for (int c = threadIdx.x; c < 2 * 4 * 32; c += blockDim.x) {
        const int isk = c >> 7, k = (c >> 5) & 3, ln = c & 31;
        const uint32_t pl = m.lane[ln];
        float4 w4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if ((pl & kLmActive) && (isk ? a.hk : a.hq) > 0) {
            const int v = k < 2 ? (int)(pl & kLmFirst) : (int)((pl >> kLmSecondShift) & kLmFirst);
            const uint16_t* w =
                reinterpret_cast<const uint16_t*>(isk ? a.k_weight : a.q_weight) + v * 8 + (k & 1) * 4;
            w4 = make_float4(act_to_f<H16>(w[0]), act_to_f<H16>(w[1]), act_to_f<H16>(w[2]),
                             act_to_f<H16>(w[3]));
        }
        wsm[c] = w4;
    }
    __syncwarp();
    int64_t t = warp_id / cpt;
    int chunk = (int)(warp_id - t * cpt);
    if (lane == 0) {  // first ring of items
        int64_t tt = t;
        int cc = chunk;
        for (int s = 0; s < stages && s < n_local; ++s) {
            issue(tt, cc, s);
            tt += dt;
            cc += dchunk;
            if (cc >= cpt) { cc -= cpt; ++tt; }
        }
    }
    __syncthreads();  // weights

    const float inv_d = 1.0f / (float)D;
    // the item `stages` ahead of the current one
    int64_t t_ahead = t, chunk_ahead = chunk;
    for (int s = 0; s < stages; ++s) {
        t_ahead += dt;
        chunk_ahead += dchunk;
        if (chunk_ahead >= cpt) { chunk_ahead -= cpt; ++t_ahead; }
    }

    int stage = 0;
    uint32_t phase = 0;
    int64_t i = 0;
    bool aborted = false;
    for (; i < n_local; ++i) {
        const bool ok = mbar_wait_bounded(&full[stage], phase, a.wait_limit_ns);
        if (__any_sync(0xffffffffu, !ok)) {
            aborted = true;
            break;
        }
        const unsigned char* buf = ring + (size_t)stage * sbytes;
        const unsigned char* trow = buf + (size_t)per_item * D * 2;
        const int h0 = chunk * per_item;
        float c[8], s[8];
        if (active) {
            if (IL) {
                if (rot1) smem_cos_sin4<F32, H16>(trow, 4 * v1, R / 2, c, s);
                if (rot2) smem_cos_sin4<F32, H16>(trow, 4 * v2, R / 2, c + 4, s + 4);
            } else if (across) {
                smem_cos_sin8<F32, H16>(trow, 8 * min(v1, v2), R / 2, c, s);
                if (swapped) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) s[k] = -s[k];
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int hi = u * HR + sub;  // head index inside the item
            const int hh = h0 + hi;
            const bool okh = active && hh < H;
            uint4 xa = make_uint4(0, 0, 0, 0), xb = xa;
            if (okh) {
                const uint4* v = reinterpret_cast<const uint4*>(buf + (size_t)hi * D * 2);
                xa = v[v1];
                xb = v[v2];
            }
            float2 fa[4], fb[4];
            fa[0] = act2_to_f2<H16>(xa.x); fa[1] = act2_to_f2<H16>(xa.y);
            fa[2] = act2_to_f2<H16>(xa.z); fa[3] = act2_to_f2<H16>(xa.w);
            fb[0] = act2_to_f2<H16>(xb.x); fb[1] = act2_to_f2<H16>(xb.y);
            fb[2] = act2_to_f2<H16>(xb.z); fb[3] = act2_to_f2<H16>(xb.w);
            float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                ss2 = fma2(fa[m], fa[m], ss2);
                ss2 = fma2(fb[m], fb[m], ss2);
            }
            const float ss = group_sum<GS>(ss2.x + ss2.y);
            if (!okh) continue;
            const bool isk = hh >= a.hq;
            const int head = isk ? hh - a.hq : hh;
            const float r = rsqrtf(ss * inv_d + a.eps);
            const float2 r2 = make_float2(r, r);
            const float4* w4 = wsm + (isk ? 4 * 32 : 0) + lane;
            const float4 wa0 = w4[0], wa1 = w4[32], wb0 = w4[64], wb1 = w4[96];
            fa[0] = mul2(mul2(fa[0], r2), make_float2(wa0.x, wa0.y));
            fa[1] = mul2(mul2(fa[1], r2), make_float2(wa0.z, wa0.w));
            fa[2] = mul2(mul2(fa[2], r2), make_float2(wa1.x, wa1.y));
            fa[3] = mul2(mul2(fa[3], r2), make_float2(wa1.z, wa1.w));
            fb[0] = mul2(mul2(fb[0], r2), make_float2(wb0.x, wb0.y));
            fb[1] = mul2(mul2(fb[1], r2), make_float2(wb0.z, wb0.w));
            fb[2] = mul2(mul2(fb[2], r2), make_float2(wb1.x, wb1.y));
            fb[3] = mul2(mul2(fb[3], r2), make_float2(wb1.z, wb1.w));
            float2 oa[4], ob[4];
            if (IL) {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    if (rot1) {
                        oa[m].x = fa[m].x * c[m] - fa[m].y * s[m];
                        oa[m].y = fa[m].y * c[m] + fa[m].x * s[m];
                    } else {
                        oa[m] = fa[m];
                    }
                    if (rot2) {
                        ob[m].x = fb[m].x * c[4 + m] - fb[m].y * s[4 + m];
                        ob[m].y = fb[m].y * c[4 + m] + fb[m].x * s[4 + m];
                    } else {
                        ob[m] = fb[m];
                    }
                }
            } else if (across) {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float2 c2 = make_float2(c[2 * m], c[2 * m + 1]);
                    const float2 s2 = make_float2(s[2 * m], s[2 * m + 1]);
                    const float2 ns2 = make_float2(-s[2 * m], -s[2 * m + 1]);
                    oa[m] = fma2(fa[m], c2, mul2(fb[m], ns2));
                    ob[m] = fma2(fb[m], c2, mul2(fa[m], s2));
                }
            } else {
#pragma unroll
                for (int m = 0; m < 4; ++m) { oa[m] = fa[m]; ob[m] = fb[m]; }
            }
            uint8_t* dst = isk
                ? a.k_out + ((size_t)t * a.k_out_stride + (size_t)head * D) * 2
                : a.q_out + ((size_t)t * a.q_out_stride + (size_t)head * D) * 2;
            st_v4(dst + (size_t)v1 * 16,
                  make_uint4(f2_to_act2<H16>(oa[0]), f2_to_act2<H16>(oa[1]),
                             f2_to_act2<H16>(oa[2]), f2_to_act2<H16>(oa[3])));
            st_v4(dst + (size_t)v2 * 16,
                  make_uint4(f2_to_act2<H16>(ob[0]), f2_to_act2<H16>(ob[1]),
                             f2_to_act2<H16>(ob[2]), f2_to_act2<H16>(ob[3])));
        }
        // Every lane is done with this buffer: refill it with the item a ring ahead.
        __syncwarp();
        if (lane == 0 && i + stages < n_local) {
            fence_proxy_async_smem();
            issue(t_ahead, (int)chunk_ahead, stage);
        }
        t_ahead += dt;
        chunk_ahead += dchunk;
        if (chunk_ahead >= cpt) { chunk_ahead -= cpt; ++t_ahead; }
        t += dt;
        chunk += dchunk;
        if (chunk >= cpt) { chunk -= cpt; ++t; }
        if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
        }
    }
    if (aborted && lane == 0) {
        atomicOr(&g_table_status, 1u);
        // Drain this warp's copies still in flight (bounded): items i .. i+stages-1.
        for (int64_t j = i; j < n_local && j < i + stages; ++j)
            mbar_wait_bounded(&full[j % stages], (uint32_t)((j / stages) & 1), a.wait_limit_ns);
    }
}

// Heads per item of the shared-memory kernel: about 4 KB of q/k per item.
__host__ __device__ inline int smem_item_heads(int D) {
    const int h = 4096 / (2 * D);
    return h < 4 ? 4 : (h > 64 ? 64 : h);
}

// Wait until all but the most recent of this thread's committed bulk stores
// have read their shared-memory source.
__device__ __forceinline__ void bulk_wait_read_allbut1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// Half-split pairs, any head_dim that is a multiple of 8 (<= 256), any even
// rotary_dim <= head_dim; q/k rows and outputs 16-byte aligned. Like the fast
// kernel, each warp streams items (heads of one token) through its own ring of
// shared-memory buffers with bulk copies; unlike it, lanes work on the heads
// in shared memory, so that any pairing is reachable: lane i takes the channel
// pairs i, i + 32, ... of a head ((p, p + rotary_dim/2) for p < rotary_dim/2,
// then the pass-through channels two by two), writes the results back in
// place and lane 0 bulk-stores the item's
// q and k heads. cos/sin come straight from the table in global memory (read
// before the item's copy is waited for), the weights sit in registers.
template <bool F32, bool H16>
__global__ void __launch_bounds__(kBlock) rope_table_smem(const RopeTableArgs a) {
    constexpr int kMaxPairs = 4;  // pairs per lane: head_dim <= 256
    const int D = a.head_dim, R = a.rotary_dim, half = R / 2;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = a.hq + a.hk;
    const int per_item = smem_item_heads(D);
    const int cpt = (H + per_item - 1) / per_item;  // items per token
    const int64_t items = a.num_tokens * cpt;
    const int stages = a.stages;
    const int sbytes = per_item * D * 2;

    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);  // [warps][stages]
    unsigned char* rings = smem + ((kBlock / 32) * stages * 8 + 127) / 128 * 128;
    uint64_t* full = bars + warp * stages;
    unsigned char* ring = rings + (size_t)warp * stages * sbytes;

    const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t n_local = warp_id < items ? (items - 1 - warp_id) / nwarps + 1 : 0;
    const int64_t dt = nwarps / cpt;
    const int dchunk = (int)(nwarps - dt * cpt);

    // The lane's channel pairs (fixed for every head) and their table slots:
    // pairs i, i + 32, ... of one head at a time.
    int ca[kMaxPairs], cb[kMaxPairs], slot[kMaxPairs];
    bool rot[kMaxPairs], has[kMaxPairs];
#pragma unroll
    for (int m = 0; m < kMaxPairs; ++m) {
        const int p = lane + 32 * m;
        has[m] = p < D / 2;
        rot[m] = has[m] && p < half;
        slot[m] = p;
        if (p < half) {
            ca[m] = p;
            cb[m] = p + half;
        } else {
            ca[m] = R + 2 * (p - half);
            cb[m] = ca[m] + 1;
        }
        if (!has[m]) ca[m] = cb[m] = 0;
    }

    auto issue = [&](int64_t t, int chunk, int s) {
        const int h0 = chunk * per_item, h1 = min(h0 + per_item, H);
        const int q1 = min(h1, a.hq), k0 = max(h0, a.hq);
        const uint32_t qbytes = h0 < a.hq ? (uint32_t)(q1 - h0) * D * 2 : 0;
        const uint32_t kbytes = h1 > a.hq ? (uint32_t)(h1 - k0) * D * 2 : 0;
        unsigned char* dst = ring + (size_t)s * sbytes;
        mbar_arrive_expect_tx(&full[s], qbytes + kbytes + a.stall_tx_bytes);
        if (qbytes)
            bulk_load(dst, a.q + ((size_t)t * a.q_stride + (size_t)h0 * D) * 2, qbytes, &full[s]);
        if (kbytes)
            bulk_load(dst + qbytes, a.k + ((size_t)t * a.k_stride + (size_t)(k0 - a.hq) * D) * 2,
                      kbytes, &full[s]);
    };

    if (lane == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    griddep_wait();
    griddep_launch_dependents();
    float wq[kMaxPairs][2], wk[kMaxPairs][2];
    {
        const uint16_t* qw = reinterpret_cast<const uint16_t*>(a.q_weight);
        const uint16_t* kw = reinterpret_cast<const uint16_t*>(a.k_weight);
#pragma unroll
        for (int m = 0; m < kMaxPairs; ++m) {
            const bool okq = has[m] && a.hq > 0, okk = has[m] && a.hk > 0;
            wq[m][0] = okq ? act_to_f<H16>(qw[ca[m]]) : 0.0f;
            wq[m][1] = okq ? act_to_f<H16>(qw[cb[m]]) : 0.0f;
            wk[m][0] = okk ? act_to_f<H16>(kw[ca[m]]) : 0.0f;
            wk[m][1] = okk ? act_to_f<H16>(kw[cb[m]]) : 0.0f;
        }
    }
    __syncwarp();
    int64_t t = warp_id / cpt;
    int chunk = (int)(warp_id - t * cpt);
    if (lane == 0) {
        int64_t tt = t;
        int cc = chunk;
        for (int s = 0; s < stages && s < n_local; ++s) {
            issue(tt, cc, s);
            tt += dt;
            cc += dchunk;
            if (cc >= cpt) { cc -= cpt; ++tt; }
        }
    }
    // the next item to copy in: `stages` after the first (refills run one item
    // behind, so after item i the copy of item i - 1 + stages is issued)
    int64_t t_ahead = t, chunk_ahead = chunk;
    for (int s = 0; s < stages; ++s) {
        t_ahead += dt;
        chunk_ahead += dchunk;
        if (chunk_ahead >= cpt) { chunk_ahead -= cpt; ++t_ahead; }
    }
    const float inv_d = 1.0f / (float)D;

    int stage = 0, prev_stage = stages - 1;
    uint32_t phase = 0;
    int64_t i = 0;
    bool aborted = false;
    for (; i < n_local; ++i) {
        // This token's cos/sin for the lane's rotated pairs, before the wait.
        float c[kMaxPairs], s[kMaxPairs];
#pragma unroll
        for (int m = 0; m < kMaxPairs; ++m) {
            c[m] = 1.0f;
            s[m] = 0.0f;
            if (rot[m]) {
                const int j = slot[m];
                if (F32) {
                    const float* tr = reinterpret_cast<const float*>(a.table) + (size_t)t * R;
                    c[m] = __ldg(tr + j);
                    s[m] = __ldg(tr + half + j);
                } else {
                    const uint16_t* tr = reinterpret_cast<const uint16_t*>(a.table) + (size_t)t * R;
                    c[m] = act_to_f<H16>(__ldg(tr + j));
                    s[m] = act_to_f<H16>(__ldg(tr + half + j));
                }
            }
        }
        const bool ok = mbar_wait_bounded(&full[stage], phase, a.wait_limit_ns);
        if (__any_sync(0xffffffffu, !ok)) {
            aborted = true;
            break;
        }
        unsigned char* buf = ring + (size_t)stage * sbytes;
        const int h0 = chunk * per_item, h1 = min(h0 + per_item, H);
        for (int hh = h0; hh < h1; ++hh) {
            uint16_t* x = reinterpret_cast<uint16_t*>(buf + (size_t)(hh - h0) * D * 2);
            const bool isk = hh >= a.hq;
            float xa[kMaxPairs], xb[kMaxPairs];
            float ss = 0.0f;
#pragma unroll
            for (int m = 0; m < kMaxPairs; ++m) {
                xa[m] = has[m] ? act_to_f<H16>(x[ca[m]]) : 0.0f;
                xb[m] = has[m] ? act_to_f<H16>(x[cb[m]]) : 0.0f;
                ss = fmaf(xa[m], xa[m], ss);
                ss = fmaf(xb[m], xb[m], ss);
            }
            const float r = rsqrtf(warp_sum(ss) * inv_d + a.eps);
#pragma unroll
            for (int m = 0; m < kMaxPairs; ++m) {
                if (!has[m]) continue;
                const float ya = xa[m] * r * (isk ? wk[m][0] : wq[m][0]);
                const float yb = xb[m] * r * (isk ? wk[m][1] : wq[m][1]);
                x[ca[m]] = f_to_act<H16>(ya * c[m] - yb * s[m]);
                x[cb[m]] = f_to_act<H16>(yb * c[m] + ya * s[m]);
            }
        }
        fence_proxy_async_smem();  // each lane's writes, before the bulk engine reads them
        __syncwarp();
        if (lane == 0) {
            // The item's results leave by bulk stores; the buffer of the
            // previous item (whose stores were issued one item ago) is refilled.
            const int q1 = min(h1, a.hq), k0 = max(h0, a.hq);
            const uint32_t qbytes = h0 < a.hq ? (uint32_t)(q1 - h0) * D * 2 : 0;
            const uint32_t kbytes = h1 > a.hq ? (uint32_t)(h1 - k0) * D * 2 : 0;
            if (qbytes)
                bulk_store(a.q_out + ((size_t)t * a.q_out_stride + (size_t)h0 * D) * 2, buf, qbytes);
            if (kbytes)
                bulk_store(a.k_out + ((size_t)t * a.k_out_stride + (size_t)(k0 - a.hq) * D) * 2,
                           buf + qbytes, kbytes);
            bulk_commit();
            if (i >= 1 && i - 1 + stages < n_local) {
                bulk_wait_read_allbut1();
                issue(t_ahead, (int)chunk_ahead, prev_stage);
            }
        }
        if (i >= 1) {
            t_ahead += dt;
            chunk_ahead += dchunk;
            if (chunk_ahead >= cpt) { chunk_ahead -= cpt; ++t_ahead; }
        }
        t += dt;
        chunk += dchunk;
        if (chunk >= cpt) { chunk -= cpt; ++t; }
        prev_stage = stage;
        if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
        }
    }
    if (lane == 0) {
        if (aborted) {
            atomicOr(&g_table_status, 1u);
            // Copies that may be in flight (bounded): items i .. i+stages-2, or
            // the whole first ring if none was consumed.
            const int64_t hi = i == 0 ? stages : i + stages - 1;
            for (int64_t j = i; j < n_local && j < hi; ++j)
                mbar_wait_bounded(&full[j % stages], (uint32_t)((j / stages) & 1), a.wait_limit_ns);
        }
        bulk_wait_all();
    }
}

// Lanes per head (gs) and 16-byte vectors per lane (mv <= 4) for adjacent
// pairs in shared memory: the split of a head's D/8 vectors that leaves the
// fewest lanes idle (then the fewest vectors per lane).
__host__ __device__ inline void il_lane_split(int D, int* gs, int* mv) {
    const int vph = D / 8;
    int best = 1 << 30;
    for (int g = 1; g <= 32; g <<= 1) {
        const int m = (vph + g - 1) / g;
        if (m > 4) continue;
        const int key = (g * m - vph) * 8 + m;
        if (key < best) {
            best = key;
            *gs = g;
            *mv = m;
        }
    }
}

// Shared-memory bytes ahead of the rings of rope_table_smem_il: mbarriers,
// fp32 weights [q | k][256], and per warp the item's cos/sin [2][128] fp32.
__host__ __device__ inline int smem_il_fixed_bytes(int stages) {
    return ((kBlock / 32) * stages * 8 + 127) / 128 * 128 + 2 * 256 * 4 + (kBlock / 32) * 2 * 128 * 4;
}

// Adjacent pairs, any head_dim that is a multiple of 8 (<= 256) and any even
// rotary_dim, q/k rows and outputs 16-byte aligned. The ring of bulk copies,
// the in-place results and the bulk stores are those of rope_table_smem; the
// work split differs: a head is a group of gs lanes and lane l of the group
// holds the 16-byte vectors l, l + gs, ... (mv of them, il_lane_split), so
// that 32/gs heads move per step with few idle lanes (head_dim 72: 4 lanes of
// 3 vectors, 8 heads per step). Weights sit in shared memory as fp32; an
// item's cos/sin are read from the table once per warp (before the item's
// copy is waited for) and staged in shared memory, where lanes of the same
// position read the same words.
// HS: half-split pairs with rotary_dim a multiple of 8 in the same layout:
// chunk c of a head is pairs 4c..4c+3, i.e. channels 4c..4c+3 and
// rotary_dim/2 + 4c..+3 (two 8-byte pieces) while 4c < rotary_dim/2, and the
// pass-through channels 8c..8c+7 (one 16-byte vector) after that.
template <bool HS, bool F32, bool H16>
__global__ void __launch_bounds__(kBlock) rope_table_smem_il(const RopeTableArgs a) {
    const int D = a.head_dim, R = a.rotary_dim, half = R / 2;
    const int vph = D / 8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = a.hq + a.hk;
    const int per_item = smem_item_heads(D);
    const int cpt = (H + per_item - 1) / per_item;  // items per token
    const int64_t items = a.num_tokens * cpt;
    const int stages = a.stages;
    const int sbytes = per_item * D * 2;
    int gs = 32, mv = 1;
    il_lane_split(D, &gs, &mv);
    const int l = lane % gs, sub = lane / gs, hps = 32 / gs;

    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);  // [warps][stages]
    float* wsm = reinterpret_cast<float*>(smem + ((kBlock / 32) * stages * 8 + 127) / 128 * 128);
    float* csm = wsm + 2 * 256 + warp * 2 * 128;  // this warp's [cos | sin] of the item
    unsigned char* rings = smem + smem_il_fixed_bytes(stages);
    uint64_t* full = bars + warp * stages;
    unsigned char* ring = rings + (size_t)warp * stages * sbytes;

    const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t n_local = warp_id < items ? (items - 1 - warp_id) / nwarps + 1 : 0;
    const int64_t dt = nwarps / cpt;
    const int dchunk = (int)(nwarps - dt * cpt);

    auto issue = [&](int64_t t, int chunk, int s) {
        const int h0 = chunk * per_item, h1 = min(h0 + per_item, H);
        const int q1 = min(h1, a.hq), k0 = max(h0, a.hq);
        const uint32_t qbytes = h0 < a.hq ? (uint32_t)(q1 - h0) * D * 2 : 0;
        const uint32_t kbytes = h1 > a.hq ? (uint32_t)(h1 - k0) * D * 2 : 0;
        unsigned char* dst = ring + (size_t)s * sbytes;
        mbar_arrive_expect_tx(&full[s], qbytes + kbytes + a.stall_tx_bytes);
        if (qbytes)
            bulk_load(dst, a.q + ((size_t)t * a.q_stride + (size_t)h0 * D) * 2, qbytes, &full[s]);
        if (kbytes)
            bulk_load(dst + qbytes, a.k + ((size_t)t * a.k_stride + (size_t)(k0 - a.hq) * D) * 2,
                      kbytes, &full[s]);
    };

    if (lane == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    griddep_wait();
    griddep_launch_dependents();
    for (int c = threadIdx.x; c < 2 * 256; c += blockDim.x) {
        const bool isk = c >= 256;
        const int cc = isk ? c - 256 : c;
        const uint16_t* w = reinterpret_cast<const uint16_t*>(isk ? a.k_weight : a.q_weight);
        wsm[c] = (cc < D && (isk ? a.hk : a.hq) > 0) ? act_to_f<H16>(w[cc]) : 0.0f;
    }
    int64_t t = warp_id / cpt;
    int chunk = (int)(warp_id - t * cpt);
    if (lane == 0) {
        int64_t tt = t;
        int cc = chunk;
        for (int s = 0; s < stages && s < n_local; ++s) {
            issue(tt, cc, s);
            tt += dt;
            cc += dchunk;
            if (cc >= cpt) { cc -= cpt; ++tt; }
        }
    }
    __syncthreads();  // weights
    // the next item to copy in (refills run one item behind)
    int64_t t_ahead = t, chunk_ahead = chunk;
    for (int s = 0; s < stages; ++s) {
        t_ahead += dt;
        chunk_ahead += dchunk;
        if (chunk_ahead >= cpt) { chunk_ahead -= cpt; ++t_ahead; }
    }
    const float inv_d = 1.0f / (float)D;

    int stage = 0, prev_stage = stages - 1;
    uint32_t phase = 0;
    int64_t i = 0;
    bool aborted = false;
    for (; i < n_local; ++i) {
        // This token's cos/sin, slots lane, lane + 32, ..., read before the wait.
        float cr[4], sr[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = lane + 32 * u;
            cr[u] = 1.0f;
            sr[u] = 0.0f;
            if (j < half) {
                if (F32) {
                    const float* tr = reinterpret_cast<const float*>(a.table) + (size_t)t * R;
                    cr[u] = __ldg(tr + j);
                    sr[u] = __ldg(tr + half + j);
                } else {
                    const uint16_t* tr = reinterpret_cast<const uint16_t*>(a.table) + (size_t)t * R;
                    cr[u] = act_to_f<H16>(__ldg(tr + j));
                    sr[u] = act_to_f<H16>(__ldg(tr + half + j));
                }
            }
        }
        const bool ok = mbar_wait_bounded(&full[stage], phase, a.wait_limit_ns);
        if (__any_sync(0xffffffffu, !ok)) {
            aborted = true;
            break;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = lane + 32 * u;
            if (j < half) {
                csm[j] = cr[u];
                csm[128 + j] = sr[u];
            }
        }
        __syncwarp();
        unsigned char* buf = ring + (size_t)stage * sbytes;
        const int h0 = chunk * per_item, h1 = min(h0 + per_item, H);
        for (int hb = h0; hb < h1; hb += hps) {  // the same trip count in every lane
            const int hh = hb + sub;
            const bool okh = hh < h1;
            uint4* head = reinterpret_cast<uint4*>(buf) + (size_t)(hh - h0) * vph;
            float2 f[4][4];
            float ss = 0.0f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int vv = l + gs * m;
                const bool here = m < mv && okh && vv < vph;
                if (HS && 4 * vv < half) {  // (a, b) of pairs 4vv..4vv+3
                    const uint16_t* h16 = reinterpret_cast<const uint16_t*>(head);
                    uint2 xa = make_uint2(0, 0), xb = xa;
                    if (here) {
                        xa = *reinterpret_cast<const uint2*>(h16 + 4 * vv);
                        xb = *reinterpret_cast<const uint2*>(h16 + half + 4 * vv);
                    }
                    const float2 a01 = act2_to_f2<H16>(xa.x), a23 = act2_to_f2<H16>(xa.y);
                    const float2 b01 = act2_to_f2<H16>(xb.x), b23 = act2_to_f2<H16>(xb.y);
                    f[m][0] = make_float2(a01.x, b01.x);
                    f[m][1] = make_float2(a01.y, b01.y);
                    f[m][2] = make_float2(a23.x, b23.x);
                    f[m][3] = make_float2(a23.y, b23.y);
                } else {
                    uint4 xv = make_uint4(0, 0, 0, 0);
                    if (here) xv = head[vv];
                    f[m][0] = act2_to_f2<H16>(xv.x);
                    f[m][1] = act2_to_f2<H16>(xv.y);
                    f[m][2] = act2_to_f2<H16>(xv.z);
                    f[m][3] = act2_to_f2<H16>(xv.w);
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) ss = fmaf(f[m][k].x, f[m][k].x, fmaf(f[m][k].y, f[m][k].y, ss));
            }
            for (int o = gs >> 1; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (!okh) continue;
            const float r = rsqrtf(ss * inv_d + a.eps);
            const float* wrow = wsm + (hh >= a.hq ? 256 : 0);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int vv = l + gs * m;
                if (m >= mv || vv >= vph) continue;
                const bool split = HS && 4 * vv < half;  // a rotated half-split chunk
                float4 w0, w1;
                if (split) {  // weights of channels 4vv.. (a) and half + 4vv.. (b)
                    const float4 wa = reinterpret_cast<const float4*>(wrow)[vv];
                    const float4 wb = reinterpret_cast<const float4*>(wrow + half)[vv];
                    w0 = make_float4(wa.x, wb.x, wa.y, wb.y);
                    w1 = make_float4(wa.z, wb.z, wa.w, wb.w);
                } else {
                    w0 = reinterpret_cast<const float4*>(wrow)[2 * vv];
                    w1 = reinterpret_cast<const float4*>(wrow)[2 * vv + 1];
                }
                const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                float4 c4 = make_float4(1.0f, 1.0f, 1.0f, 1.0f), s4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (4 * vv < half) {
                    c4 = reinterpret_cast<const float4*>(csm)[vv];
                    s4 = reinterpret_cast<const float4*>(csm + 128)[vv];
                }
                const float cv[4] = {c4.x, c4.y, c4.z, c4.w}, sv[4] = {s4.x, s4.y, s4.z, s4.w};
                uint32_t o32[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const bool rk = HS ? split : 4 * vv + k < half;
                    const float ya = f[m][k].x * r * wv[2 * k], yb = f[m][k].y * r * wv[2 * k + 1];
                    const float c = rk ? cv[k] : 1.0f, s = rk ? sv[k] : 0.0f;
                    o32[k] = f2_to_act2<H16>(make_float2(ya * c - yb * s, yb * c + ya * s));
                }
                if (split) {  // o32[k] = (a_k, b_k): regroup into the a and b pieces
                    uint16_t* h16 = reinterpret_cast<uint16_t*>(head);
                    *reinterpret_cast<uint2*>(h16 + 4 * vv) =
                        make_uint2(__byte_perm(o32[0], o32[1], 0x5410), __byte_perm(o32[2], o32[3], 0x5410));
                    *reinterpret_cast<uint2*>(h16 + half + 4 * vv) =
                        make_uint2(__byte_perm(o32[0], o32[1], 0x7632), __byte_perm(o32[2], o32[3], 0x7632));
                } else {
                    head[vv] = make_uint4(o32[0], o32[1], o32[2], o32[3]);
                }
            }
        }
        fence_proxy_async_smem();  // each lane's writes, before the bulk engine reads them
        __syncwarp();
        if (lane == 0) {
            // The item's results leave by bulk stores; the buffer of the
            // previous item (whose stores were issued one item ago) is refilled.
            const int q1 = min(h1, a.hq), k0 = max(h0, a.hq);
            const uint32_t qbytes = h0 < a.hq ? (uint32_t)(q1 - h0) * D * 2 : 0;
            const uint32_t kbytes = h1 > a.hq ? (uint32_t)(h1 - k0) * D * 2 : 0;
            if (qbytes)
                bulk_store(a.q_out + ((size_t)t * a.q_out_stride + (size_t)h0 * D) * 2, buf, qbytes);
            if (kbytes)
                bulk_store(a.k_out + ((size_t)t * a.k_out_stride + (size_t)(k0 - a.hq) * D) * 2,
                           buf + qbytes, kbytes);
            bulk_commit();
            if (i >= 1 && i - 1 + stages < n_local) {
                bulk_wait_read_allbut1();
                issue(t_ahead, (int)chunk_ahead, prev_stage);
            }
        }
        if (i >= 1) {
            t_ahead += dt;
            chunk_ahead += dchunk;
            if (chunk_ahead >= cpt) { chunk_ahead -= cpt; ++t_ahead; }
        }
        t += dt;
        chunk += dchunk;
        if (chunk >= cpt) { chunk -= cpt; ++t; }
        prev_stage = stage;
        if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
        }
    }
    if (lane == 0) {
        if (aborted) {
            atomicOr(&g_table_status, 1u);
            const int64_t hi = i == 0 ? stages : i + stages - 1;
            for (int64_t j = i; j < n_local && j < hi; ++j)
                mbar_wait_bounded(&full[j % stages], (uint32_t)((j / stages) & 1), a.wait_limit_ns);
        }
        bulk_wait_all();
    }
}

// One warp per head; any head_dim <= 256, any even rotary_dim <= head_dim,
// 2-byte alignment. The normalised head goes through shared memory so that
// every lane can read its partner channel.
template <bool F32, bool H16>
__global__ void __launch_bounds__(kBlock) rope_table_general(const RopeTableArgs a) {
    __shared__ float ybuf[kBlock / 32][256];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int D = a.head_dim, R = a.rotary_dim, half = R / 2;
    const int H = a.hq + a.hk;
    const int64_t ngroups = a.num_tokens * H;
    float* y = ybuf[warp];
    const uint16_t* qw = reinterpret_cast<const uint16_t*>(a.q_weight);
    const uint16_t* kw = reinterpret_cast<const uint16_t*>(a.k_weight);
    for (int64_t g = (int64_t)blockIdx.x * (kBlock / 32) + warp; g < ngroups;
         g += (int64_t)gridDim.x * (kBlock / 32)) {
        const int64_t t = g / H;
        const int hh = (int)(g - t * H);
        const bool isk = hh >= a.hq;
        const int head = isk ? hh - a.hq : hh;
        const uint16_t* src = reinterpret_cast<const uint16_t*>(isk ? a.k : a.q) +
                              (size_t)t * (isk ? a.k_stride : a.q_stride) + (size_t)head * D;
        uint16_t* dst = reinterpret_cast<uint16_t*>(isk ? a.k_out : a.q_out) +
                        (size_t)t * (isk ? a.k_out_stride : a.q_out_stride) + (size_t)head * D;
        const uint16_t* w = isk ? kw : qw;
        float x[8];
        float ss = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int d = lane + 32 * k;
            x[k] = d < D ? act_to_f<H16>(src[d]) : 0.0f;
            ss += x[k] * x[k];
        }
        ss = warp_sum(ss);
        const float r = rsqrtf(ss / (float)D + a.eps);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int d = lane + 32 * k;
            if (d < D) y[d] = x[k] * r * act_to_f<H16>(__ldg(w + d));
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int d = lane + 32 * k;
            if (d >= D) continue;
            float o = y[d];
            if (d < R) {
                int j, p;
                bool first;
                if (a.interleaved) {
                    j = d >> 1; first = (d & 1) == 0; p = d ^ 1;
                } else {
                    first = d < half; j = first ? d : d - half; p = first ? d + half : d - half;
                }
                float c, s;
                if (F32) {
                    const float* tr = reinterpret_cast<const float*>(a.table) + (size_t)t * R;
                    c = __ldg(tr + j); s = __ldg(tr + half + j);
                } else {
                    const uint16_t* tr = reinterpret_cast<const uint16_t*>(a.table) + (size_t)t * R;
                    c = act_to_f<H16>(__ldg(tr + j));
                    s = act_to_f<H16>(__ldg(tr + half + j));
                }
                o = first ? y[d] * c - y[p] * s : y[d] * c + y[p] * s;
            }
            dst[d] = f_to_act<H16>(o);
        }
        __syncwarp();
    }
}

template <typename K>
cudaError_t launch_persistent(K kern, int64_t work_blocks, const RopeTableArgs& a,
                              cudaStream_t stream, LaunchInfo* info, int id) {
    int sms = 0, per_sm = 0;
    cudaError_t e = cached_sm_count(&sms);
    if (e == cudaSuccess)
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), kBlock, 0, &per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)sms * per_sm,
                                                                 work_blocks));
    kern<<<grid, kBlock, 0, stream>>>(a);
    if (info) {
        info->grid = grid;
        info->block = kBlock;
        info->smem = 0;
        info->kernel_id = id;
    }
    return cudaGetLastError();
}

// Host side of LaneMap. The lanes of a head are l < D/16; lane l holds
// vectors (l, l + D/16) when pairs are adjacent channels, the pair
// (l, l + rotary_dim/16) when they are half split and l < rotary_dim/16, and
// two pass-through vectors otherwise. For each phase of 8 lanes (a 128-bit
// shared load serves 8 lanes at a time) every choice of load order is scored
// by its bank-group collisions over the item's 4 rounds, and the best kept.
LaneMap make_lane_map(const RopeTableArgs& a, int GS) {
    const int D = a.head_dim, R = a.rotary_dim;
    const int L = D / 16, VPH = D / 8, HR = 32 / GS, r16 = R / 16, rv = R / 8;
    int va[32], vb[32];
    bool act[32], acr[32];
    for (int ln = 0; ln < 32; ++ln) {
        const int l = ln % GS;
        act[ln] = l < L;
        acr[ln] = false;
        va[ln] = vb[ln] = 0;
        if (!act[ln]) continue;
        if (a.interleaved) {
            va[ln] = l; vb[ln] = l + L;
        } else if (l < r16) {
            va[ln] = l; vb[ln] = l + r16; acr[ln] = true;
        } else {
            va[ln] = rv + 2 * (l - r16); vb[ln] = va[ln] + 1;
        }
    }
    uint32_t order = 0;  // bit ln: lane ln loads (vb, va)
    for (int ph = 0; ph < 4; ++ph) {
        int best = 1 << 30, best_bits = 0;
        for (int bits = 0; bits < 256; ++bits) {
            int cost = 0;
            for (int u = 0; u < kUnroll; ++u) {
                for (int ld = 0; ld < 2; ++ld) {
                    int count[8] = {0, 0, 0, 0, 0, 0, 0, 0}, worst = 0;
                    for (int j = 0; j < 8; ++j) {
                        const int ln = ph * 8 + j;
                        if (!act[ln]) continue;
                        const bool sw = (bits >> j) & 1;
                        const int v = (ld == 0) != sw ? va[ln] : vb[ln];
                        const int hi = u * HR + ln / GS;
                        const int c = ++count[(hi * VPH + v) & 7];
                        worst = c > worst ? c : worst;
                    }
                    cost += worst;
                }
            }
            cost = cost * 16 + __builtin_popcount(bits);  // fewer swaps on a tie
            if (cost < best) {
                best = cost;
                best_bits = bits;
            }
        }
        order |= (uint32_t)best_bits << (8 * ph);
    }
    LaneMap m;
    for (int ln = 0; ln < 32; ++ln) {
        if (!act[ln]) {
            m.lane[ln] = 0;
            continue;
        }
        const bool sw = (order >> ln) & 1;
        const int v1 = sw ? vb[ln] : va[ln], v2 = sw ? va[ln] : vb[ln];
        uint32_t w = (uint32_t)v1 | ((uint32_t)v2 << kLmSecondShift) | kLmActive;
        if (acr[ln]) w |= kLmAcross | (sw ? kLmSwapped : 0u);
        if (a.interleaved && v1 < rv) w |= kLmRot1;
        if (a.interleaved && v2 < rv) w |= kLmRot2;
        m.lane[ln] = w;
    }
    return m;
}

// make_lane_map is a search (about 65 thousand steps); launches look up its
// result per shape.
LaneMap lane_map_cached(const RopeTableArgs& a, int GS) {
    static std::mutex mu;
    static std::unordered_map<uint32_t, LaneMap> cache;
    const uint32_t key = (uint32_t)a.head_dim | ((uint32_t)a.rotary_dim << 9) |
                         ((uint32_t)(a.interleaved != 0) << 18) | ((uint32_t)GS << 19);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    const LaneMap m = make_lane_map(a, GS);
    cache.emplace(key, m);
    return m;
}

template <typename K>
cudaError_t launch_bulk(K kern, const RopeTableArgs& a0, int per_item, cudaStream_t stream,
                        LaunchInfo* info, int id) {
    RopeTableArgs a = a0;
    const int tb = a.table_f32 ? 4 : 2;
    const int sbytes = table_stage_bytes(per_item, a.head_dim, a.rotary_dim, tb);
    const int warps = kBlock / 32;
    // Two CTAs per SM, each warp with as many ring buffers (2..4) as fit.
    const int fixed = kWsmBytes + 128 + warps * 4 * 8;
    a.stages = std::max(2, std::min(4, (227 * 1024 / 2 - 1024 - fixed) / (warps * sbytes)));
    if (a.wait_limit_ns == 0) a.wait_limit_ns = 2000000000ull;  // 2 s
    const int smem = kWsmBytes + ((warps * a.stages * 8 + 127) / 128 * 128) +
                     warps * a.stages * sbytes;
    int sms = 0, per_sm = 0;
    cudaError_t e = cached_sm_count(&sms);
    if (e == cudaSuccess)
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), kBlock, smem, &per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int H = a.hq + a.hk;
    const int64_t items = a.num_tokens * ((H + per_item - 1) / per_item);
    const int64_t want_blocks = (items + warps - 1) / warps;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)sms * per_sm,
                                                                 want_blocks));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kBlock);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const LaneMap m = lane_map_cached(a, 32 / (per_item / kUnroll));
    e = cudaLaunchKernelEx(&cfg, kern, a, m);
    if (e != cudaSuccess) {
        cudaGetLastError();
        forget_kernel(reinterpret_cast<const void*>(kern));
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), kBlock, smem, &per_sm);
        if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, kern, a, m);
    }
    if (info) {
        info->grid = grid;
        info->block = kBlock;
        info->smem = smem;
        info->kernel_id = id;
    }
    return e;
}

template <typename K>
cudaError_t launch_smem(K kern, bool il, const RopeTableArgs& a0, cudaStream_t stream,
                        LaunchInfo* info, int id) {
    RopeTableArgs a = a0;
    const int sbytes = smem_item_heads(a.head_dim) * a.head_dim * 2;
    const int warps = kBlock / 32;
    // Two CTAs per SM, each warp with as many ring buffers (2..4) as fit.
    auto fixed_bytes = [&](int stages) {
        return il ? smem_il_fixed_bytes(stages) : ((warps * stages * 8 + 127) / 128 * 128);
    };
    a.stages = std::max(2, std::min(4, (227 * 1024 / 2 - 1024 - fixed_bytes(4)) / (warps * sbytes)));
    if (a.wait_limit_ns == 0) a.wait_limit_ns = 2000000000ull;  // 2 s
    const int smem = fixed_bytes(a.stages) + warps * a.stages * sbytes;
    int sms = 0, per_sm = 0;
    cudaError_t e = cached_sm_count(&sms);
    if (e == cudaSuccess)
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), kBlock, smem, &per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int per_item = smem_item_heads(a.head_dim);
    const int64_t items = a.num_tokens * ((a.hq + a.hk + per_item - 1) / per_item);
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>((int64_t)sms * per_sm, (items + warps - 1) / warps));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kBlock);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) {
        cudaGetLastError();
        forget_kernel(reinterpret_cast<const void*>(kern));
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), kBlock, smem, &per_sm);
        if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, kern, a);
    }
    if (info) {
        info->grid = grid;
        info->block = kBlock;
        info->smem = smem;
        info->kernel_id = id;
    }
    return e;
}

// Whether the shared-memory kernel takes these arguments: head_dim a multiple
// of 8 and every q/k row (input and output) on a 16-byte boundary.
bool smem_path_ok(const RopeTableArgs& a) {
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (a.head_dim % 8 != 0 || a.head_dim > 256) return false;
    if (a.hq > 0 && !(al(a.q) && al(a.q_out) && a.q_stride % 8 == 0 && a.q_out_stride % 8 == 0))
        return false;
    if (a.hk > 0 && !(al(a.k) && al(a.k_out) && a.k_stride % 8 == 0 && a.k_out_stride % 8 == 0))
        return false;
    return true;
}

template <int GS, bool H16>
cudaError_t run_fast_act(const RopeTableArgs& a, cudaStream_t stream, LaunchInfo* info) {
    const int per_item = kUnroll * (32 / GS);
    const int id = 1000 + (H16 ? 500 : 0) + GS * 10 + (a.interleaved ? 1 : 0) * 2 +
                   (a.table_f32 ? 1 : 0);
    if (a.interleaved) {
        return a.table_f32
            ? launch_bulk(rope_table_bulk<GS, true, true, H16>, a, per_item, stream, info, id)
            : launch_bulk(rope_table_bulk<GS, true, false, H16>, a, per_item, stream, info, id);
    }
    return a.table_f32
        ? launch_bulk(rope_table_bulk<GS, false, true, H16>, a, per_item, stream, info, id)
        : launch_bulk(rope_table_bulk<GS, false, false, H16>, a, per_item, stream, info, id);
}

template <int GS>
cudaError_t run_fast(const RopeTableArgs& a, cudaStream_t stream, LaunchInfo* info) {
    return a.act_f16 ? run_fast_act<GS, true>(a, stream, info)
                     : run_fast_act<GS, false>(a, stream, info);
}

}  // namespace

cudaError_t launch_rope_table(const RopeTableArgs& a, int fast_path, cudaStream_t stream,
                              LaunchInfo* info) {
    if (fast_path) {
        const int L = a.head_dim / 16;
        if (L <= 1) return run_fast<1>(a, stream, info);
        if (L <= 2) return run_fast<2>(a, stream, info);
        if (L <= 4) return run_fast<4>(a, stream, info);
        if (L <= 8) return run_fast<8>(a, stream, info);
        return run_fast<16>(a, stream, info);
    }
    if (smem_path_ok(a)) {
        const int id = 2100 + (a.interleaved ? 100 : 0) + (a.act_f16 ? 10 : 0) + (a.table_f32 ? 1 : 0);
        // Adjacent pairs always take the vector split (measured faster at every
        // head_dim tried, 72 to 192). Half split takes it only when rotary_dim
        // is a multiple of 8 and a head's pairs do not fill whole warps; with a
        // multiple of 32 pairs the pairwise lanes are busy and measured faster.
        const bool pairwise = !a.interleaved &&
                              (a.rotary_dim % 8 != 0 || (a.head_dim / 2) % 32 == 0);
        if (pairwise) {
            if (a.act_f16) {
                return a.table_f32 ? launch_smem(rope_table_smem<true, true>, false, a, stream, info, id)
                                   : launch_smem(rope_table_smem<false, true>, false, a, stream, info, id);
            }
            return a.table_f32 ? launch_smem(rope_table_smem<true, false>, false, a, stream, info, id)
                               : launch_smem(rope_table_smem<false, false>, false, a, stream, info, id);
        }
        if (a.interleaved) {
            if (a.act_f16) {
                return a.table_f32
                    ? launch_smem(rope_table_smem_il<false, true, true>, true, a, stream, info, id)
                    : launch_smem(rope_table_smem_il<false, false, true>, true, a, stream, info, id);
            }
            return a.table_f32
                ? launch_smem(rope_table_smem_il<false, true, false>, true, a, stream, info, id)
                : launch_smem(rope_table_smem_il<false, false, false>, true, a, stream, info, id);
        }
        if (a.rotary_dim % 8 == 0) {  // half split in 8-byte pieces
            const int idv = id + 50;
            if (a.act_f16) {
                return a.table_f32
                    ? launch_smem(rope_table_smem_il<true, true, true>, true, a, stream, info, idv)
                    : launch_smem(rope_table_smem_il<true, false, true>, true, a, stream, info, idv);
            }
            return a.table_f32
                ? launch_smem(rope_table_smem_il<true, true, false>, true, a, stream, info, idv)
                : launch_smem(rope_table_smem_il<true, false, false>, true, a, stream, info, idv);
        }
        if (a.act_f16) {
            return a.table_f32 ? launch_smem(rope_table_smem<true, true>, false, a, stream, info, id)
                               : launch_smem(rope_table_smem<false, true>, false, a, stream, info, id);
        }
        return a.table_f32 ? launch_smem(rope_table_smem<true, false>, false, a, stream, info, id)
                           : launch_smem(rope_table_smem<false, false>, false, a, stream, info, id);
    }
    const int64_t groups = a.num_tokens * (a.hq + a.hk);
    const int64_t blocks = (groups + kBlock / 32 - 1) / (kBlock / 32);
    if (a.act_f16) {
        return a.table_f32
            ? launch_persistent(rope_table_general<true, true>, blocks, a, stream, info, 2011)
            : launch_persistent(rope_table_general<false, true>, blocks, a, stream, info, 2010);
    }
    return a.table_f32
        ? launch_persistent(rope_table_general<true, false>, blocks, a, stream, info, 2001)
        : launch_persistent(rope_table_general<false, false>, blocks, a, stream, info, 2000);
}

cudaError_t read_table_status(uint32_t* out, int clear, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_table_status, sizeof(uint32_t), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && clear) {
        const uint32_t zero = 0;
        e = cudaMemcpyToSymbolAsync(g_table_status, &zero, sizeof(uint32_t), 0,
                                    cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    }
    return e;
}

}  // namespace qknr
