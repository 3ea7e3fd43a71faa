// Packed-QKV across-heads RMSNorm + 3D RoPE + V copy (+ FP8 E4M3 output).
//
// Computes the operation of "flashinfer.norm.fused_qk_rmsnorm_rope" (FlashInfer
// API docs; summary, Parameters, Returns) in one pass over HBM: every input
// byte is read once, every output byte written once, nothing else touches
// memory.
//
// Thread layout. One token is worked on by a group of threads. A slot is
// (head, l): the two 16-byte vectors l and l + D/16 of one Q or K head. The
// pipelined kernel deals a token's slots -- all Q slots, then all K slots --
// to the group's threads S at a time (thread i takes slots i, i + Bg, ...), so
// that Q and K head counts that differ (grouped-query attention) still give
// every thread the same work; the fallback kernel gives a thread S Q slots and
// the S K slots of the same index. Either way l = thread mod D/16, the same
// for all of a thread's slots.
// Vector l's channel e pairs with vector l + D/16's channel e in NeoX mode; in
// interleaved mode adjacent channels of one vector pair up. Either way the 8
// rotation pairs of a thread stay inside the thread, at fixed pair slots.
//
// Per token: sum x^2 of Q and of K over the group (warp shuffles, one shared
// exchange, one barrier), then scale, rotate, convert and store.
//
// cos/sin: the frequency of pair slot j, base^(-2i/C) / 2pi, is kept as a
// 64-bit binary fraction of a turn; pos * fraction modulo 2^64 is the exact
// angle in turns, so no precision is lost at large positions. A shared table
// holds cos/sin of every (axis, position, frequency) -- at most
// ppf*Cf/2 + pph*Ch/2 + ppw*Cw/2 entries -- built once per CTA; when it would
// not fit, the angles are evaluated per token instead.
//
// rope3d_mg_kernel (the fast path): one persistent CTA per SM runs G
// independent token pipelines ("groups"), each with its own named barrier and
// its own ring of shared-memory row buffers that bulk asynchronous copies (the
// TMA engine, one instruction per row, tracked by mbarriers) fill ahead of
// use. The angle table and the norm weights (converted once to fp32, laid out
// for conflict-free reads) are shared by all groups. Threads keep no row data
// in registers across the per-token barrier: they read their vectors from the
// ring before it (for sum x^2) and again after it (to scale and rotate), which
// keeps registers low enough for ~24 warps per SM. The group's first thread
// refills a buffer one token later, once every thread has passed the next
// barrier, and in bf16 mode copies V straight from the ring to v_out with a
// bulk store. Every wait on a copy is bounded in time; on expiry the group
// votes through its barrier, raises bit 0 of a device status word, drains its
// own copies and leaves.
//
// rope3d_reg_kernel (fallback for rows too large for the ring): 128-bit
// loads straight into registers.
#include "common.cuh"
#include "launch.h"
#include "launch_cache.h"

#include <algorithm>

namespace qknr {

__device__ unsigned int g_rope3d_status;

namespace {

constexpr int kMaxBlock = 512;
constexpr int kMaxTableBytes = 64 * 1024;
constexpr int kSmemPerSm = 227 * 1024;

// Frequencies of the D/2 pair slots and, if enabled, the cos/sin table.
template <int D>
__device__ __forceinline__ void setup_angles(const Rope3DArgs& a, uint64_t* gq, float2* tab) {
    constexpr int HALF = D / 2;
    const int tid = threadIdx.x, B = blockDim.x;
    const int hcf = a.cf >> 1, hch = a.ch >> 1, hcw = a.cw >> 1;
    for (int j = tid; j < HALF; j += B) {
        int i, C;
        if (j < hcf) {
            i = j; C = a.cf;
        } else if (j < hcf + hch) {
            i = j - hcf; C = a.ch;
        } else {
            i = j - hcf - hch; C = a.cw;
        }
        gq[j] = turns_q64(a.base, i, C);
    }
    __syncthreads();
    if (a.use_table) {
        const int nf = a.ppf * hcf, nh = a.pph * hch;
        for (int e = tid; e < a.table_entries; e += B) {
            int pos, j;
            if (e < nf) {
                pos = e / hcf; j = e - pos * hcf;
            } else if (e < nf + nh) {
                const int r = e - nf;
                pos = r / hch; j = hcf + (r - pos * hch);
            } else {
                const int r = e - nf - nh;
                pos = r / hcw; j = hcf + hch + (r - pos * hcw);
            }
            float s, c;
            turn_sincos((uint32_t)pos, gq[j], &s, &c);
            tab[e] = make_float2(c, s);
        }
    }
}

// cos/sin of an integer position for a stored frequency, out of line so that
// the table path carries none of its code.
__device__ __noinline__ float2 direct_cos_sin(uint32_t pos, uint64_t turns) {
    float s, c;
    turn_sincos(pos, turns, &s, &c);
    return make_float2(c, s);
}

// cos/sin of pair slot j for patch (pf, ph, pw).
__device__ __forceinline__ float2 pair_cos_sin(const Rope3DArgs& a, const uint64_t* gq,
                                               const float2* tab, int j, int pf, int ph, int pw) {
    const int hcf = a.cf >> 1, hch = a.ch >> 1, hcw = a.cw >> 1;
    int pos, col, base;
    if (j < hcf) {
        pos = pf; col = j; base = pf * hcf;
    } else if (j < hcf + hch) {
        pos = ph; col = j - hcf; base = a.ppf * hcf + ph * hch;
    } else {
        pos = pw; col = j - hcf - hch; base = a.ppf * hcf + a.pph * hch + pw * hcw;
    }
    if (a.use_table) return tab[base + col];
    return direct_cos_sin((uint32_t)pos, gq[j]);
}

// Row vectors of a thread's two slot halves, as (va, dv): the first half is
// vector va of the head, the second vector va + dv. Whole-head NeoX and
// interleaved pairs: vectors l and l + D/16. NeoX per axis group: the thread's
// pair slots 8l..8l+7 lie in one axis group (the groups are multiples of 16
// channels), with first channel o and C channels, and slot 8l + e pairs
// channels o + i and o + C/2 + i (i = 8l + e - o/2): vectors o/16 + l and
// o/16 + C/16 + l. The slots keep their frequencies, so cos/sin are unchanged.
template <int D, bool NEOX>
__device__ __forceinline__ void slot_vectors(const Rope3DArgs& a, int l, int& va, int& dv) {
    va = l;
    dv = D / 16;
    if (NEOX && a.neox_per_axis) {
        const int j0 = 8 * l, hcf = a.cf >> 1, hch = a.ch >> 1;
        const int o = j0 < hcf ? 0 : (j0 < hcf + hch ? a.cf : a.cf + a.ch);
        const int C = j0 < hcf ? a.cf : (j0 < hcf + hch ? a.ch : a.cw);
        va = o / 16 + l;
        dv = C / 16;
    }
}

// Scale by r * weight, rotate the thread's 8 pairs, convert, store one slot.
// Channel pairs travel as float2 so that the scaling (and the NeoX rotation,
// whose partners sit in the two vectors) use the packed fp32x2 instructions.
template <int D, bool NEOX, bool FP8>
__device__ __forceinline__ void apply_slot(const uint4& va, const uint4& vb, const uint4& wva,
                                           const uint4& wvb, bool norm, float r,
                                           const float (&cs)[8], const float (&sn)[8],
                                           uint8_t* out_head, int l, float scale) {
    constexpr int L = D / 16;
    float2 xa[4] = {bf16x2_to_f2(va.x), bf16x2_to_f2(va.y), bf16x2_to_f2(va.z),
                    bf16x2_to_f2(va.w)};
    float2 xb[4] = {bf16x2_to_f2(vb.x), bf16x2_to_f2(vb.y), bf16x2_to_f2(vb.z),
                    bf16x2_to_f2(vb.w)};
    if (norm) {
        const float2 r2 = make_float2(r, r);
        const float2 wa[4] = {bf16x2_to_f2(wva.x), bf16x2_to_f2(wva.y), bf16x2_to_f2(wva.z),
                              bf16x2_to_f2(wva.w)};
        const float2 wb[4] = {bf16x2_to_f2(wvb.x), bf16x2_to_f2(wvb.y), bf16x2_to_f2(wvb.z),
                              bf16x2_to_f2(wvb.w)};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            xa[m] = mul2(mul2(xa[m], r2), wa[m]);
            xb[m] = mul2(mul2(xb[m], r2), wb[m]);
        }
    }
    float2 oa[4], ob[4];
    if constexpr (NEOX) {
        // channel e of vector a pairs with channel e of vector b, slot e
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float2 c = make_float2(cs[2 * m], cs[2 * m + 1]);
            const float2 sv = make_float2(sn[2 * m], sn[2 * m + 1]);
            const float2 nsv = make_float2(-sn[2 * m], -sn[2 * m + 1]);
            oa[m] = fma2(xa[m], c, mul2(xb[m], nsv));
            ob[m] = fma2(xb[m], c, mul2(xa[m], sv));
        }
    } else {
        // channels (2m, 2m+1) of a vector pair up, slot m (vector a) or 4+m (b)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            oa[m].x = xa[m].x * cs[m] - xa[m].y * sn[m];
            oa[m].y = xa[m].y * cs[m] + xa[m].x * sn[m];
            ob[m].x = xb[m].x * cs[4 + m] - xb[m].y * sn[4 + m];
            ob[m].y = xb[m].y * cs[4 + m] + xb[m].x * sn[4 + m];
        }
    }
    if constexpr (FP8) {
        const float fa[8] = {oa[0].x, oa[0].y, oa[1].x, oa[1].y, oa[2].x, oa[2].y, oa[3].x, oa[3].y};
        const float fb[8] = {ob[0].x, ob[0].y, ob[1].x, ob[1].y, ob[2].x, ob[2].y, ob[3].x, ob[3].y};
        uint8_t* p = out_head + 8 * l;
        st_v2(p, pack8_e4m3(fa, scale));
        st_v2(p + 8 * L, pack8_e4m3(fb, scale));
    } else {
        uint8_t* p = out_head + 16 * l;
        st_v4(p, make_uint4(f2_to_bf16x2(oa[0]), f2_to_bf16x2(oa[1]), f2_to_bf16x2(oa[2]),
                            f2_to_bf16x2(oa[3])));
        st_v4(p + 16 * L, make_uint4(f2_to_bf16x2(ob[0]), f2_to_bf16x2(ob[1]),
                                     f2_to_bf16x2(ob[2]), f2_to_bf16x2(ob[3])));
    }
}

// As apply_slot, with the weights of the slot given as fp32 from shared
// memory: w points at float4 index (h*2 + m)*VPH + v for vector v, half m.
// For E4M3 output the caller has already folded the output scale into r (or,
// without the norm, into cos/sin).
template <int D, bool NEOX, bool FP8>
__device__ __forceinline__ void apply_slot_wf(const uint4& va, const uint4& vb,
                                              const float4* wsm_head, bool norm, float r,
                                              const float (&cs)[8], const float (&sn)[8],
                                              uint8_t* out_head, int l) {
    constexpr int L = D / 16;
    constexpr int VPH = D / 8;
    float2 xa[4] = {bf16x2_to_f2(va.x), bf16x2_to_f2(va.y), bf16x2_to_f2(va.z),
                    bf16x2_to_f2(va.w)};
    float2 xb[4] = {bf16x2_to_f2(vb.x), bf16x2_to_f2(vb.y), bf16x2_to_f2(vb.z),
                    bf16x2_to_f2(vb.w)};
    if (norm) {
        const float2 r2 = make_float2(r, r);
        const float4 a0 = wsm_head[l], a1 = wsm_head[VPH + l];
        const float4 b0 = wsm_head[l + L], b1 = wsm_head[VPH + l + L];
        const float2 wa[4] = {make_float2(a0.x, a0.y), make_float2(a0.z, a0.w),
                              make_float2(a1.x, a1.y), make_float2(a1.z, a1.w)};
        const float2 wb[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w),
                              make_float2(b1.x, b1.y), make_float2(b1.z, b1.w)};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            xa[m] = mul2(mul2(xa[m], r2), wa[m]);
            xb[m] = mul2(mul2(xb[m], r2), wb[m]);
        }
    }
    float2 oa[4], ob[4];
    if constexpr (NEOX) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float2 c = make_float2(cs[2 * m], cs[2 * m + 1]);
            const float2 sv = make_float2(sn[2 * m], sn[2 * m + 1]);
            const float2 nsv = make_float2(-sn[2 * m], -sn[2 * m + 1]);
            oa[m] = fma2(xa[m], c, mul2(xb[m], nsv));
            ob[m] = fma2(xb[m], c, mul2(xa[m], sv));
        }
    } else {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            oa[m].x = xa[m].x * cs[m] - xa[m].y * sn[m];
            oa[m].y = xa[m].y * cs[m] + xa[m].x * sn[m];
            ob[m].x = xb[m].x * cs[4 + m] - xb[m].y * sn[4 + m];
            ob[m].y = xb[m].y * cs[4 + m] + xb[m].x * sn[4 + m];
        }
    }
    if constexpr (FP8) {
        const float fa[8] = {oa[0].x, oa[0].y, oa[1].x, oa[1].y, oa[2].x, oa[2].y, oa[3].x, oa[3].y};
        const float fb[8] = {ob[0].x, ob[0].y, ob[1].x, ob[1].y, ob[2].x, ob[2].y, ob[3].x, ob[3].y};
        uint8_t* p = out_head + 8 * l;
        st_v2(p, pack8_e4m3_unscaled(fa));
        st_v2(p + 8 * L, pack8_e4m3_unscaled(fb));
    } else {
        uint8_t* p = out_head + 16 * l;
        st_v4(p, make_uint4(f2_to_bf16x2(oa[0]), f2_to_bf16x2(oa[1]), f2_to_bf16x2(oa[2]),
                            f2_to_bf16x2(oa[3])));
        st_v4(p + 16 * L, make_uint4(f2_to_bf16x2(ob[0]), f2_to_bf16x2(ob[1]),
                                     f2_to_bf16x2(ob[2]), f2_to_bf16x2(ob[3])));
    }
}

// Sum of squares of the 16 channels of a vector pair (even channels in .x,
// odd ones in .y), straight from the bf16 pairs.
__device__ __forceinline__ float2 ssq_pair(const uint4& va, const uint4& vb, float2 acc) {
    const uint32_t w[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
    for (int m = 0; m < 8; ++m) acc = ssq_bf16x2(w[m], acc);
    return acc;
}

// Pair slots of vector pair (l, l + D/16): NeoX -> 8l..8l+7; interleaved ->
// 4l..4l+3 and 4(l + D/16)..+3.
template <int D, bool NEOX>
__device__ __forceinline__ int slot_of(int l, int k) {
    constexpr int L = D / 16;
    return NEOX ? 8 * l + k : (k < 4 ? 4 * l + k : 4 * (l + L) + (k - 4));
}

template <int S>
__device__ __forceinline__ void load_weights(const Rope3DArgs& a, int VPH, int L, int l, int tid,
                                             int B, uint4 (&wqa)[S], uint4 (&wqb)[S],
                                             uint4 (&wka)[S], uint4 (&wkb)[S]) {
    const int nq = a.hq * L, nk = a.hk * L;
    const bool norm = a.is_qk_norm != 0;
#pragma unroll
    for (int i = 0; i < S; ++i) {
        const int slot = tid + i * B;
        const uint4 one = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        wqa[i] = wqb[i] = wka[i] = wkb[i] = one;
        if (norm && slot < nq) {
            const uint4* w = reinterpret_cast<const uint4*>(a.q_weight) + (slot / L) * VPH + l;
            wqa[i] = w[0]; wqb[i] = w[L];
        }
        if (norm && slot < nk) {
            const uint4* w = reinterpret_cast<const uint4*>(a.k_weight) + (slot / L) * VPH + l;
            wka[i] = w[0]; wkb[i] = w[L];
        }
    }
}

// ---------------------------------------------------------------------------
// Pipelined kernel: G token pipelines per CTA, sharing the angle table and
// the fp32 weights.
// ---------------------------------------------------------------------------
constexpr int kCsPitch = 20;  // floats per l-row of the staged cos/sin (16 + pad)
constexpr int kMaxGroups = 15;

// Shared-memory layout of the pipelined kernel, in bytes from the base.
struct MgLayout {
    int ring, full, cst, red, abort, wts, gq, tab, total;
};

__host__ __device__ inline MgLayout mg_layout(int D, int groups, int stages, int row_bytes,
                                              int weight_floats, int table_bytes) {
    MgLayout o;
    const int L = D / 16, HALF = D / 2;
    o.ring = 0;
    o.full = groups * stages * row_bytes;
    o.cst = (o.full + 8 * groups * stages + 15) & ~15;
    o.red = o.cst + groups * 2 * L * kCsPitch * 4;
    o.abort = o.red + groups * 64 * 8;
    o.wts = o.abort + 16;
    o.gq = o.wts + weight_floats * 4;
    o.tab = o.gq + HALF * 8;
    o.total = o.tab + table_bytes;
    return o;
}

// S slots per thread. MIXED: thread i takes slots i, i + Bg, ... of the list
// [Q slots | K slots]; otherwise slot k of a thread stands for the Q slot and
// the K slot of index i + k * Bg (equal Q and K head counts).
template <int D, bool NEOX, bool FP8, int S, bool MIXED>
__global__ void __launch_bounds__(768, 1) rope3d_mg_kernel(const Rope3DArgs a) {
    constexpr int L = D / 16;
    constexpr int VPH = D / 8;
    constexpr int HALF = D / 2;
    constexpr int OUTB = FP8 ? 1 : 2;

    const int G = a.groups;
    const int Bg = blockDim.x / G;  // threads per group, a multiple of 32
    const bool partial = a.mode == kModePartialSsq;  // sums of squares only
    const bool supplied = a.mode == kModeSuppliedSsq;  // sums come from ssq_in
    const int row_bytes = (a.hq + a.hk + a.hv) * D * 2;  // token stride in qkv
    // A partial pass needs only the Q and K part of each row.
    const int stage_bytes = partial ? (a.hq + a.hk) * D * 2 : row_bytes;
    const int stages = a.stages;
    const bool norm = a.is_qk_norm != 0;
    const MgLayout lay = mg_layout(D, G, stages, stage_bytes,
                                   (norm && !partial) ? (a.hq + a.hk) * D : 0,
                                   a.use_table ? a.table_entries * 8 : 0);
    extern __shared__ __align__(128) unsigned char smem[];
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + lay.abort);
    float4* wsm = reinterpret_cast<float4*>(smem + lay.wts);
    uint64_t* gq = reinterpret_cast<uint64_t*>(smem + lay.gq);
    float2* tab = reinterpret_cast<float2*>(smem + lay.tab);

    const int tid = threadIdx.x;
    const int g = tid / Bg;
    const int ctid = tid - g * Bg;
    unsigned char* ring = smem + lay.ring + (size_t)g * stages * stage_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.full) + g * stages;
    float* cst = reinterpret_cast<float*>(smem + lay.cst) + g * 2 * L * kCsPitch;
    float2* red = reinterpret_cast<float2*>(smem + lay.red) + g * 64;

    const int64_t NP = (int64_t)gridDim.x * G;  // pipelines in the grid
    const uint32_t tx = (uint32_t)stage_bytes + a.stall_tx_bytes;
    const int vbytes = partial ? 0 : a.hv * D * 2;
    const bool v_bulk = a.v_bulk && vbytes > 0;
    const size_t v_off = (size_t)(a.hq + a.hk) * D * 2;  // V inside a row

    // Everything up to griddep_wait() touches only shared memory and the
    // arguments, so with a programmatic dependent launch it overlaps the end
    // of the previous kernel on the stream.
    if (tid == 0) {
        for (int q = 0; q < G * stages; ++q)
            mbar_init(reinterpret_cast<uint64_t*>(smem + lay.full) + q, 1);
        *abort_flag = 0u;
        fence_mbar_init();
        griddep_wait();
        // First `stages` rows of every pipeline.
        for (int q = 0; q < G; ++q) {
            const int64_t p = (int64_t)blockIdx.x * G + q;
            unsigned char* rq = smem + lay.ring + (size_t)q * stages * stage_bytes;
            uint64_t* fq = reinterpret_cast<uint64_t*>(smem + lay.full) + q * stages;
            for (int i = 0; i < stages && p + i * NP < a.num_tokens; ++i) {
                mbar_arrive_expect_tx(&fq[i], tx);
                bulk_load(rq + (size_t)i * stage_bytes, a.qkv + (p + i * NP) * row_bytes,
                          stage_bytes, &fq[i]);
            }
        }
    }
    // Partial sums of warps a group does not have stay zero.
    for (int q = tid; q < G * 64; q += blockDim.x)
        reinterpret_cast<float2*>(smem + lay.red)[q] = make_float2(0.0f, 0.0f);
    if (!partial) setup_angles<D>(a, gq, tab);
    griddep_wait();
    griddep_launch_dependents();
    if (norm && !partial) {
        // fp32 weights, float4 index (h*2 + m)*VPH + v for channels 8v+4m..+3 of head h.
        const int nq4 = a.hq * VPH * 2, n4 = (a.hq + a.hk) * VPH * 2;
        for (int q = tid; q < n4; q += blockDim.x) {
            const bool isk = q >= nq4;
            const int r = isk ? q - nq4 : q;
            const int h = r / (2 * VPH), m = (r / VPH) & 1, v = r % VPH;
            const uint2 w = reinterpret_cast<const uint2*>(isk ? a.k_weight : a.q_weight)
                [((size_t)h * VPH + v) * 2 + m];
            wsm[q] = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
        }
    }
    __syncthreads();

    // ------------------------------ one pipeline ------------------------------
    const int64_t p = (int64_t)blockIdx.x * G + g;
    const int64_t n_local = p < a.num_tokens ? (a.num_tokens - 1 - p) / NP + 1 : 0;
    const int lane = tid & 31, cwarp = ctid >> 5, nwarps = Bg >> 5;
    const int l = ctid % L;
    const int nq = a.hq * L, nk = a.hk * L, nv = a.hv * VPH;

    // Patch of the current token, stepped by the pipeline stride without division.
    const int hw = a.pph * a.ppw;
    const int P = a.ppf * hw;
    int pf, ph, pw, df, dh, dw;
    {
        const int s0 = (int)((p + a.pos_offset) % P);
        pf = s0 / hw; ph = (s0 - pf * hw) / a.ppw; pw = s0 - pf * hw - ph * a.ppw;
        const int st = (int)(NP % P);
        df = st / hw; dh = (st - df * hw) / a.ppw; dw = st - df * hw - dh * a.ppw;
    }
    // Staging: thread ctid < HALF owns pair slot j = ctid each token. Its
    // destination in the staged cos/sin rows, its axis and its column in the
    // table are fixed: packed into one word (dst 11 bits, axis 2, column 8).
    const int hcf = a.cf >> 1, hch = a.ch >> 1, hcw = a.cw >> 1;
    const int nf = a.ppf * hcf, nh = a.pph * hch;
    uint32_t stage_code = 0;
    if (HALF <= Bg && ctid < HALF) {
        const int j = ctid;
        int rl, k;
        if (NEOX) {
            rl = j >> 3; k = j & 7;
        } else if (j < 4 * L) {
            rl = j >> 2; k = j & 3;
        } else {
            rl = (j - 4 * L) >> 2; k = 4 + ((j - 4 * L) & 3);
        }
        const int axis = j < hcf ? 0 : (j < hcf + hch ? 1 : 2);
        const int col = axis == 0 ? j : (axis == 1 ? j - hcf : j - hcf - hch);
        stage_code = (uint32_t)(rl * kCsPitch + k) | ((uint32_t)axis << 11) | ((uint32_t)col << 13);
    }
    const float inv_nq = 1.0f / (float)(a.norm_q_elems > 0 ? a.norm_q_elems : 1);
    const float inv_nk = 1.0f / (float)(a.norm_k_elems > 0 ? a.norm_k_elems : 1);
    const int vout_bytes = a.hv * D * OUTB;

    int64_t i = 0;
    bool aborted = false;
    // Ring position of token i (i mod stages), the phase its buffer is in
    // ((i / stages) mod 2), and the previous token's buffer, kept by counting.
    int stage = 0, prev_stage = stages - 1;
    uint32_t phase = 0;
    int64_t t = p;
    for (; i < n_local; ++i, t += NP) {
        const int parity = (int)(i & 1);
        const bool ok = mbar_wait_abortable(&full[stage], phase, a.wait_limit_ns, abort_flag);
        const unsigned char* row = ring + (size_t)stage * stage_bytes;
        if (ctid == 0 && ok && v_bulk) {
            bulk_store(a.v_out + t * vbytes, row + v_off, (uint32_t)vbytes);
            bulk_commit();
        }
        float2 sq2 = make_float2(0.0f, 0.0f), sk2 = make_float2(0.0f, 0.0f);
        if (ok) {
            if (norm && !supplied) {
#pragma unroll
                for (int k = 0; k < S; ++k) {
                    const int slot = ctid + k * Bg;
                    if constexpr (MIXED) {  // Q slots, then K slots
                        if (slot < nq) {
                            const uint4* q4 =
                                reinterpret_cast<const uint4*>(row) + (slot / L) * VPH + l;
                            sq2 = ssq_pair(q4[0], q4[L], sq2);
                        } else if (slot < nq + nk) {
                            const uint4* k4 = reinterpret_cast<const uint4*>(row) +
                                              (a.hq + (slot - nq) / L) * VPH + l;
                            sk2 = ssq_pair(k4[0], k4[L], sk2);
                        }
                    } else {
                        const int h = slot / L;
                        if (slot < nq) {
                            const uint4* q4 = reinterpret_cast<const uint4*>(row) + h * VPH + l;
                            sq2 = ssq_pair(q4[0], q4[L], sq2);
                        }
                        if (slot < nk) {
                            const uint4* k4 =
                                reinterpret_cast<const uint4*>(row) + (a.hq + h) * VPH + l;
                            sk2 = ssq_pair(k4[0], k4[L], sk2);
                        }
                    }
                }
            }
            if (!v_bulk && !partial) {
                const unsigned char* vrow = row + v_off;
                uint8_t* vout = a.v_out + t * vout_bytes;
                const float2 vs2 = make_float2(a.v_scale, a.v_scale);
                for (int vi = ctid; vi < nv; vi += Bg) {
                    const uint4 v = reinterpret_cast<const uint4*>(vrow)[vi];
                    if constexpr (FP8) {
                        const float2 f0 = mul2(bf16x2_to_f2(v.x), vs2);
                        const float2 f1 = mul2(bf16x2_to_f2(v.y), vs2);
                        const float2 f2 = mul2(bf16x2_to_f2(v.z), vs2);
                        const float2 f3 = mul2(bf16x2_to_f2(v.w), vs2);
                        const float f[8] = {f0.x, f0.y, f1.x, f1.y, f2.x, f2.y, f3.x, f3.y};
                        st_v2(vout + (size_t)vi * 8, pack8_e4m3_unscaled(f));
                    } else {
                        st_v4(vout + (size_t)vi * 16, v);
                    }
                }
            }
        }
        // This token's cos/sin, staged per l-row: [c_0..c_7][s_0..s_7][pad].
        if (!partial) {
            float* cp = cst + parity * L * kCsPitch;
            if (HALF <= Bg) {
                if (ctid < HALF) {  // whole warps: HALF is a multiple of 32
                    const int axis = (stage_code >> 11) & 3;
                    const int col = (int)(stage_code >> 13);
                    float2 v;
                    if (a.use_table) {
                        const int base = axis == 0 ? pf * hcf
                                                   : (axis == 1 ? nf + ph * hch : nf + nh + pw * hcw);
                        v = tab[base + col];
                    } else {
                        const int pos = axis == 0 ? pf : (axis == 1 ? ph : pw);
                        v = direct_cos_sin((uint32_t)pos, gq[ctid]);
                    }
                    const int dst = (int)(stage_code & 2047);
                    cp[dst] = v.x;
                    cp[dst + 8] = v.y;
                }
            } else {
                for (int j = ctid; j < HALF; j += Bg) {
                    int rl, k;
                    if (NEOX) {
                        rl = j >> 3; k = j & 7;
                    } else if (j < 4 * L) {
                        rl = j >> 2; k = j & 3;
                    } else {
                        rl = (j - 4 * L) >> 2; k = 4 + ((j - 4 * L) & 3);
                    }
                    const float2 v = pair_cos_sin(a, gq, tab, j, pf, ph, pw);
                    cp[rl * kCsPitch + k] = v.x;
                    cp[rl * kCsPitch + 8 + k] = v.y;
                }
            }
        }
        if (norm && !supplied) {
            const float sq = warp_sum(sq2.x + sq2.y);
            const float sk = warp_sum(sk2.x + sk2.y);
            if (lane == 0) red[parity * 32 + cwarp] = make_float2(sq, sk);
        }
        if (named_barrier_or(1 + g, Bg, !ok)) {
            aborted = true;
            if (ctid == 0) *abort_flag = 1u;
            break;
        }
        // Every thread of the group is past token i-1 (it re-reads token i's
        // rows after this barrier, not i-1's): refill i-1's buffer with the
        // token `stages` after it. A second barrier at the end of each token
        // would free the buffer earlier, but it stops warps from running
        // ahead and measured slower.
        if (ctid == 0 && i >= 1 && i - 1 + stages < n_local) {
            if (v_bulk) bulk_wait_read_all();
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&full[prev_stage], tx);
            bulk_load(ring + (size_t)prev_stage * stage_bytes,
                      a.qkv + (t + (stages - 1) * NP) * row_bytes, stage_bytes, &full[prev_stage]);
        }
        prev_stage = stage;
        if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
        }
        pw += dw;
        ph += dh + (pw >= a.ppw ? 1 : 0);
        pw -= pw >= a.ppw ? a.ppw : 0;
        pf += df + (ph >= a.pph ? 1 : 0);
        ph -= ph >= a.pph ? a.pph : 0;
        pf -= pf >= a.ppf ? a.ppf : 0;

        float rq = 1.0f, rk = 1.0f;
        if (norm) {
            float tq, tk;
            if (supplied) {  // sums over every slice's heads, from the caller
                const float2 v = reinterpret_cast<const float2*>(a.ssq_in)[t];
                tq = v.x; tk = v.y;
            } else {
                // (sum Q^2, sum K^2) partials of the warps, two warps per 16-byte read
                const float4* r4 = reinterpret_cast<const float4*>(red + parity * 32);
                float4 acc = r4[0];
                for (int w = 1; w < (nwarps + 1) >> 1; ++w) {
                    const float4 v = r4[w];
                    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
                }
                tq = acc.x + acc.z; tk = acc.y + acc.w;
            }
            if (partial) {  // this slice's sums are the whole result
                if (ctid == 0) reinterpret_cast<float2*>(a.ssq_out)[t] = make_float2(tq, tk);
                continue;
            }
            rq = rsqrtf(tq * inv_nq + a.eps);
            rk = rsqrtf(tk * inv_nk + a.eps);
            if (FP8) {  // E4M3(value * scale): the scale rides on r
                rq *= a.q_scale;
                rk *= a.q_scale;
            }
        }
        float cs[8], sn[8];
        {
            const float4* cp = reinterpret_cast<const float4*>(cst + (parity * L + l) * kCsPitch);
            const float4 c0 = cp[0], c1 = cp[1], s0 = cp[2], s1 = cp[3];
            cs[0] = c0.x; cs[1] = c0.y; cs[2] = c0.z; cs[3] = c0.w;
            cs[4] = c1.x; cs[5] = c1.y; cs[6] = c1.z; cs[7] = c1.w;
            sn[0] = s0.x; sn[1] = s0.y; sn[2] = s0.z; sn[3] = s0.w;
            sn[4] = s1.x; sn[5] = s1.y; sn[6] = s1.z; sn[7] = s1.w;
            if (FP8 && !norm) {  // no r to carry the scale: put it on cos/sin
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    cs[k] *= a.q_scale;
                    sn[k] *= a.q_scale;
                }
            }
        }
#pragma unroll
        for (int k = 0; k < S; ++k) {
            const int slot = ctid + k * Bg;
            const bool is_q = slot < nq;
            const bool is_k = MIXED ? (slot >= nq && slot < nq + nk) : slot < nk;
            const int hq_i = slot / L, hk_i = MIXED ? (slot - nq) / L : slot / L;
            if (is_q) {
                const uint4* q4 = reinterpret_cast<const uint4*>(row) + hq_i * VPH + l;
                apply_slot_wf<D, NEOX, FP8>(q4[0], q4[L], wsm + hq_i * 2 * VPH, norm, rq, cs, sn,
                                            a.q_out + (t * a.hq + hq_i) * D * OUTB, l);
            }
            if (is_k) {
                const uint4* k4 = reinterpret_cast<const uint4*>(row) + (a.hq + hk_i) * VPH + l;
                apply_slot_wf<D, NEOX, FP8>(k4[0], k4[L], wsm + (a.hq + hk_i) * 2 * VPH, norm,
                                            rk, cs, sn, a.k_out + (t * a.hk + hk_i) * D * OUTB,
                                            l);
            }
        }
    }
    if (ctid == 0) {
        if (aborted || *abort_flag) {
            atomicOr(&g_rope3d_status, 1u);
            // Drain this pipeline's loads that may still be in flight (bounded):
            // tokens i .. i+stages-2 (refills run one token behind), or the
            // whole first ring if nothing was consumed yet.
            const int64_t hi = i == 0 ? stages : i + stages - 1;
            for (int64_t j = i; j < n_local && j < hi; ++j)
                mbar_wait_bounded(&full[j % stages], (uint32_t)((j / stages) & 1),
                                  a.wait_limit_ns);
        }
        if (v_bulk) bulk_wait_all();
    }
}

// ---------------------------------------------------------------------------
// Register-resident pipelined kernel: as rope3d_mg_kernel (G token pipelines
// per CTA, bulk-copy rings, shared angle table), but each thread keeps its NS
// slots in registers, as loaded (bf16 pairs), from the sums of squares
// (mixed-precision FMAs on the pairs) to the stores. With equal Q and K head
// counts the weights stay bf16 in shared memory and x * w is a mixed-precision
// product too; with grouped-query heads they are widened to fp32 once. A token
// therefore needs NS/2 times fewer threads, every slot is read from shared
// memory once and widened once, and the token's own ring buffer is free at
// the token's barrier: it is refilled there, one and a half tokens of copy
// time ahead of its next use. The per-token work
// that every warp repeats (the wait, the reductions, the barrier, r, the
// cos/sin reads, the loop) is spread over NS slots per thread instead of two.
//
// Slots of a thread: without MIXED, slots k < NS/2 are the Q slots
// ctid + k*Bg and slots NS/2 + k the K slots of the same indices (equal Q and
// K head counts); with MIXED, slot k is entry ctid + k*Bg of the list
// [Q slots | K slots]. Either way l = ctid mod D/16 for all of them.
// ---------------------------------------------------------------------------
template <int NS>
constexpr int rr_max_threads() {
    return NS >= 4 ? 384 : 768;
}

template <int D, bool NEOX, bool FP8, int NS, bool MIXED>
__global__ void __launch_bounds__(rr_max_threads<NS>(), 1) rope3d_rr_kernel(const Rope3DArgs a) {
    constexpr int L = D / 16;
    constexpr int VPH = D / 8;
    constexpr int HALF = D / 2;
    constexpr int OUTB = FP8 ? 1 : 2;
    constexpr int S = NS / 2;
    // Weights in shared memory as stored (bf16, [head][D], multiplied with
    // mixed-precision FMAs) for equal Q and K head counts; as fp32 pairs
    // ([head][2][VPH] float4) for grouped-query heads, where the bf16 form
    // measured slower.
    constexpr bool BW = !MIXED;

    const int G = a.groups;
    const int Bg = blockDim.x / G;
    const int row_bytes = (a.hq + a.hk + a.hv) * D * 2;
    const int stages = a.stages;
    const bool norm = a.is_qk_norm != 0;
    const bool supplied = a.mode == kModeSuppliedSsq;  // sums come from ssq_in
    const MgLayout lay = mg_layout(D, G, stages, row_bytes,
                                   norm ? (a.hq + a.hk) * D / (BW ? 2 : 1) : 0,
                                   a.use_table ? a.table_entries * 8 : 0);
    extern __shared__ __align__(128) unsigned char smem[];
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + lay.abort);
    float4* wsm = reinterpret_cast<float4*>(smem + lay.wts);
    uint4* wsb = reinterpret_cast<uint4*>(smem + lay.wts);
    uint64_t* gq = reinterpret_cast<uint64_t*>(smem + lay.gq);
    float2* tab = reinterpret_cast<float2*>(smem + lay.tab);

    const int tid = threadIdx.x;
    const int g = tid / Bg;
    const int ctid = tid - g * Bg;
    unsigned char* ring = smem + lay.ring + (size_t)g * stages * row_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.full) + g * stages;
    float* cst = reinterpret_cast<float*>(smem + lay.cst) + g * 2 * L * kCsPitch;
    float2* red = reinterpret_cast<float2*>(smem + lay.red) + g * 64;

    const int64_t NP = (int64_t)gridDim.x * G;
    const uint32_t tx = (uint32_t)row_bytes + a.stall_tx_bytes;
    const int vbytes = a.hv * D * 2;
    const bool v_bulk = a.v_bulk && vbytes > 0;
    const size_t v_off = (size_t)(a.hq + a.hk) * D * 2;

    // Up to griddep_wait() only shared memory and the arguments are touched.
    if (tid == 0) {
        for (int q = 0; q < G * stages; ++q)
            mbar_init(reinterpret_cast<uint64_t*>(smem + lay.full) + q, 1);
        *abort_flag = 0u;
        fence_mbar_init();
        griddep_wait();
        for (int q = 0; q < G; ++q) {
            const int64_t p = (int64_t)blockIdx.x * G + q;
            unsigned char* rq = smem + lay.ring + (size_t)q * stages * row_bytes;
            uint64_t* fq = reinterpret_cast<uint64_t*>(smem + lay.full) + q * stages;
            for (int i = 0; i < stages && p + i * NP < a.num_tokens; ++i) {
                mbar_arrive_expect_tx(&fq[i], tx);
                bulk_load(rq + (size_t)i * row_bytes, a.qkv + (p + i * NP) * row_bytes,
                          row_bytes, &fq[i]);
            }
        }
    }
    for (int q = tid; q < G * 64; q += blockDim.x)
        reinterpret_cast<float2*>(smem + lay.red)[q] = make_float2(0.0f, 0.0f);
    setup_angles<D>(a, gq, tab);
    griddep_wait();
    griddep_launch_dependents();
    if (norm && BW) {  // Q heads, then K heads
        const int nq16 = a.hq * VPH, n16 = (a.hq + a.hk) * VPH;
        for (int q = tid; q < n16; q += blockDim.x)
            wsb[q] = q < nq16 ? reinterpret_cast<const uint4*>(a.q_weight)[q]
                              : reinterpret_cast<const uint4*>(a.k_weight)[q - nq16];
    } else if (norm) {
        const int nq4 = a.hq * VPH * 2, n4 = (a.hq + a.hk) * VPH * 2;
        for (int q = tid; q < n4; q += blockDim.x) {
            const bool isk = q >= nq4;
            const int r = isk ? q - nq4 : q;
            const int h = r / (2 * VPH), m = (r / VPH) & 1, v = r % VPH;
            const uint2 w = reinterpret_cast<const uint2*>(isk ? a.k_weight : a.q_weight)
                [((size_t)h * VPH + v) * 2 + m];
            wsm[q] = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
        }
    }
    __syncthreads();

    const int64_t p = (int64_t)blockIdx.x * G + g;
    const int64_t n_local = p < a.num_tokens ? (a.num_tokens - 1 - p) / NP + 1 : 0;
    const int lane = tid & 31, cwarp = ctid >> 5, nwarps = Bg >> 5;
    const int l = ctid % L;
    int va, dv;  // the row vectors of the thread's slot halves
    slot_vectors<D, NEOX>(a, l, va, dv);
    const int nq = a.hq * L, nk = a.hk * L, nv = a.hv * VPH;

    // The thread's slots: the row vector of their first half (uint4 index in a
    // row, -1 for none), their head's weights (uint4 index in wsb or float4
    // index in wsm), their
    // byte offset in the output token row, and whether they are Q slots.
    int roff[NS], woff[NS], ooff[NS];
    bool isq[NS];
#pragma unroll
    for (int k = 0; k < NS; ++k) {
        bool q, valid;
        int hh;
        if constexpr (MIXED) {
            const int idx = ctid + k * Bg;
            q = idx < nq;
            valid = idx < nq + nk;
            hh = q ? idx / L : (idx - nq) / L;
        } else {
            q = k < S;
            const int idx = ctid + (q ? k : k - S) * Bg;
            valid = idx < (q ? nq : nk);
            hh = idx / L;
        }
        const int hg = q ? hh : a.hq + hh;
        isq[k] = q;
        roff[k] = valid ? hg * VPH + va : -1;
        woff[k] = BW ? hg * VPH : hg * 2 * VPH;
        ooff[k] = hh * D * OUTB + (FP8 ? 8 : 16) * va;
    }

    // Patch of the current token, stepped by the pipeline stride.
    const int hw = a.pph * a.ppw;
    const int P = a.ppf * hw;
    int pf, ph, pw, df, dh, dw;
    {
        const int s0 = (int)((p + a.pos_offset) % P);
        pf = s0 / hw; ph = (s0 - pf * hw) / a.ppw; pw = s0 - pf * hw - ph * a.ppw;
        const int st = (int)(NP % P);
        df = st / hw; dh = (st - df * hw) / a.ppw; dw = st - df * hw - dh * a.ppw;
    }
    const int hcf = a.cf >> 1, hch = a.ch >> 1, hcw = a.cw >> 1;
    const int nf = a.ppf * hcf, nh = a.pph * hch;
    uint32_t stage_code = 0;
    if (HALF <= Bg && ctid < HALF) {
        const int j = ctid;
        int rl, k;
        if (NEOX) {
            rl = j >> 3; k = j & 7;
        } else if (j < 4 * L) {
            rl = j >> 2; k = j & 3;
        } else {
            rl = (j - 4 * L) >> 2; k = 4 + ((j - 4 * L) & 3);
        }
        const int axis = j < hcf ? 0 : (j < hcf + hch ? 1 : 2);
        const int col = axis == 0 ? j : (axis == 1 ? j - hcf : j - hcf - hch);
        stage_code = (uint32_t)(rl * kCsPitch + k) | ((uint32_t)axis << 11) | ((uint32_t)col << 13);
    }
    const float inv_nq = 1.0f / (float)(a.norm_q_elems > 0 ? a.norm_q_elems : 1);
    const float inv_nk = 1.0f / (float)(a.norm_k_elems > 0 ? a.norm_k_elems : 1);
    const int64_t q_tok = (int64_t)a.hq * D * OUTB, k_tok = (int64_t)a.hk * D * OUTB;
    const int vout_bytes = a.hv * D * OUTB;

    int64_t i = 0;
    bool aborted = false;
    int stage = 0;
    uint32_t phase = 0;
    int64_t t = p;
    for (; i < n_local; ++i, t += NP) {
        const int parity = (int)(i & 1);
        const bool ok = mbar_wait_abortable(&full[stage], phase, a.wait_limit_ns, abort_flag);
        const unsigned char* row = ring + (size_t)stage * row_bytes;
        if (ctid == 0 && ok && v_bulk) {
            bulk_store(a.v_out + t * vbytes, row + v_off, (uint32_t)vbytes);
            bulk_commit();
        }
        uint4 px[NS][2];  // the slots' channels as loaded (bf16 pairs)
        float2 sq2 = make_float2(0.0f, 0.0f), sk2 = make_float2(0.0f, 0.0f);
        if (ok) {
#pragma unroll
            for (int k = 0; k < NS; ++k) {
                if (roff[k] < 0) continue;
                const uint4* v4 = reinterpret_cast<const uint4*>(row) + roff[k];
                px[k][0] = v4[0];
                px[k][1] = v4[dv];
                if (norm && !supplied) {
                    float2 acc = isq[k] ? sq2 : sk2;
                    const uint32_t w[8] = {px[k][0].x, px[k][0].y, px[k][0].z, px[k][0].w,
                                           px[k][1].x, px[k][1].y, px[k][1].z, px[k][1].w};
#pragma unroll
                    for (int m = 0; m < 8; ++m) acc = ssq_bf16x2(w[m], acc);
                    if (isq[k]) sq2 = acc; else sk2 = acc;
                }
            }
            if (!v_bulk) {
                const unsigned char* vrow = row + v_off;
                uint8_t* vout = a.v_out + t * vout_bytes;
                const float2 vs2 = make_float2(a.v_scale, a.v_scale);
                for (int vi = ctid; vi < nv; vi += Bg) {
                    const uint4 v = reinterpret_cast<const uint4*>(vrow)[vi];
                    if constexpr (FP8) {
                        const float2 f0 = mul2(bf16x2_to_f2(v.x), vs2);
                        const float2 f1 = mul2(bf16x2_to_f2(v.y), vs2);
                        const float2 f2 = mul2(bf16x2_to_f2(v.z), vs2);
                        const float2 f3 = mul2(bf16x2_to_f2(v.w), vs2);
                        const float f[8] = {f0.x, f0.y, f1.x, f1.y, f2.x, f2.y, f3.x, f3.y};
                        st_v2(vout + (size_t)vi * 8, pack8_e4m3_unscaled(f));
                    } else {
                        st_v4(vout + (size_t)vi * 16, v);
                    }
                }
            }
        }
        // This token's cos/sin, staged per l-row: [c_0..c_7][s_0..s_7][pad].
        {
            float* cp = cst + parity * L * kCsPitch;
            if (HALF <= Bg) {
                if (ctid < HALF) {
                    const int axis = (stage_code >> 11) & 3;
                    const int col = (int)(stage_code >> 13);
                    float2 v;
                    if (a.use_table) {
                        const int base = axis == 0 ? pf * hcf
                                                   : (axis == 1 ? nf + ph * hch : nf + nh + pw * hcw);
                        v = tab[base + col];
                    } else {
                        const int pos = axis == 0 ? pf : (axis == 1 ? ph : pw);
                        v = direct_cos_sin((uint32_t)pos, gq[ctid]);
                    }
                    const int dst = (int)(stage_code & 2047);
                    cp[dst] = v.x;
                    cp[dst + 8] = v.y;
                }
            } else {
                for (int j = ctid; j < HALF; j += Bg) {
                    int rl, k;
                    if (NEOX) {
                        rl = j >> 3; k = j & 7;
                    } else if (j < 4 * L) {
                        rl = j >> 2; k = j & 3;
                    } else {
                        rl = (j - 4 * L) >> 2; k = 4 + ((j - 4 * L) & 3);
                    }
                    const float2 v = pair_cos_sin(a, gq, tab, j, pf, ph, pw);
                    cp[rl * kCsPitch + k] = v.x;
                    cp[rl * kCsPitch + 8 + k] = v.y;
                }
            }
        }
        if (norm && !supplied) {
            const float sq = warp_sum(sq2.x + sq2.y);
            const float sk = warp_sum(sk2.x + sk2.y);
            if (lane == 0) red[parity * 32 + cwarp] = make_float2(sq, sk);
        }
        if (named_barrier_or(1 + g, Bg, !ok)) {
            aborted = true;
            if (ctid == 0) *abort_flag = 1u;
            break;
        }
        // Every thread holds this token's slots in registers and has read its
        // V: the buffer takes the token `stages` after this one.
        if (ctid == 0 && i + stages < n_local) {
            if (v_bulk) bulk_wait_read_all();
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&full[stage], tx);
            bulk_load(ring + (size_t)stage * row_bytes, a.qkv + (t + stages * NP) * row_bytes,
                      row_bytes, &full[stage]);
        }
        if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
        }
        pw += dw;
        ph += dh + (pw >= a.ppw ? 1 : 0);
        pw -= pw >= a.ppw ? a.ppw : 0;
        pf += df + (ph >= a.pph ? 1 : 0);
        ph -= ph >= a.pph ? a.pph : 0;
        pf -= pf >= a.ppf ? a.ppf : 0;

        float rq = 1.0f, rk = 1.0f;
        if (norm) {
            float tq, tk;
            if (supplied) {  // sums over every slice's heads, from the caller
                const float2 v = reinterpret_cast<const float2*>(a.ssq_in)[t];
                tq = v.x; tk = v.y;
            } else {
                const float4* r4 = reinterpret_cast<const float4*>(red + parity * 32);
                float4 acc = r4[0];
                for (int w = 1; w < (nwarps + 1) >> 1; ++w) {
                    const float4 v = r4[w];
                    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
                }
                tq = acc.x + acc.z; tk = acc.y + acc.w;
            }
            rq = rsqrtf(tq * inv_nq + a.eps);
            rk = rsqrtf(tk * inv_nk + a.eps);
        }
        if (FP8) {  // E4M3(value * scale): the scale rides on r
            rq *= a.q_scale;
            rk *= a.q_scale;
        }
        float cs[8], sn[8];
        {
            const float4* cp = reinterpret_cast<const float4*>(cst + (parity * L + l) * kCsPitch);
            const float4 c0 = cp[0], c1 = cp[1], s0 = cp[2], s1 = cp[3];
            cs[0] = c0.x; cs[1] = c0.y; cs[2] = c0.z; cs[3] = c0.w;
            cs[4] = c1.x; cs[5] = c1.y; cs[6] = c1.z; cs[7] = c1.w;
            sn[0] = s0.x; sn[1] = s0.y; sn[2] = s0.z; sn[3] = s0.w;
            sn[4] = s1.x; sn[5] = s1.y; sn[6] = s1.z; sn[7] = s1.w;
        }
        uint8_t* const qrow = a.q_out + t * q_tok;
        uint8_t* const krow = a.k_out + t * k_tok;
        // Q slots with r_q on cos/sin, then K slots with r_k: the rotation is
        // linear, so the norm factor (and the E4M3 scale) rides on it.
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
            const float r = pass == 0 ? rq : rk;
            const float2 r2 = make_float2(r, r), nr2 = make_float2(-r, -r);
            float2 C[4], Sv[4], NSv[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float2 c = make_float2(cs[2 * m], cs[2 * m + 1]);
                const float2 s = make_float2(sn[2 * m], sn[2 * m + 1]);
                C[m] = mul2(c, r2);
                Sv[m] = mul2(s, r2);
                NSv[m] = mul2(s, nr2);
            }
#pragma unroll
            for (int k = 0; k < NS; ++k) {
                if (roff[k] < 0 || isq[k] != (pass == 0)) continue;
                float2 ya[4], yb[4];
                if (norm && BW) {  // x * w, exact in fp32, from the bf16 pairs as loaded
                    const uint32_t xa[4] = {px[k][0].x, px[k][0].y, px[k][0].z, px[k][0].w};
                    const uint32_t xb[4] = {px[k][1].x, px[k][1].y, px[k][1].z, px[k][1].w};
                    const uint4 wa = wsb[woff[k] + va], wb = wsb[woff[k] + va + dv];
                    const uint32_t wa4[4] = {wa.x, wa.y, wa.z, wa.w};
                    const uint32_t wb4[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        ya[m] = mul_bf16x2(xa[m], wa4[m]);
                        yb[m] = mul_bf16x2(xb[m], wb4[m]);
                    }
                } else {
                    const float2 xs[8] = {
                        bf16x2_to_f2(px[k][0].x), bf16x2_to_f2(px[k][0].y),
                        bf16x2_to_f2(px[k][0].z), bf16x2_to_f2(px[k][0].w),
                        bf16x2_to_f2(px[k][1].x), bf16x2_to_f2(px[k][1].y),
                        bf16x2_to_f2(px[k][1].z), bf16x2_to_f2(px[k][1].w)};
                    if (norm) {
                        const float4* w = wsm + woff[k];
                        const float4 a0 = w[va], a1 = w[VPH + va], b0 = w[va + dv],
                                     b1 = w[VPH + va + dv];
                        ya[0] = mul2(xs[0], make_float2(a0.x, a0.y));
                        ya[1] = mul2(xs[1], make_float2(a0.z, a0.w));
                        ya[2] = mul2(xs[2], make_float2(a1.x, a1.y));
                        ya[3] = mul2(xs[3], make_float2(a1.z, a1.w));
                        yb[0] = mul2(xs[4], make_float2(b0.x, b0.y));
                        yb[1] = mul2(xs[5], make_float2(b0.z, b0.w));
                        yb[2] = mul2(xs[6], make_float2(b1.x, b1.y));
                        yb[3] = mul2(xs[7], make_float2(b1.z, b1.w));
                    } else {
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            ya[m] = xs[m];
                            yb[m] = xs[4 + m];
                        }
                    }
                }
                float2 oa[4], ob[4];
                if constexpr (NEOX) {
                    // channel e of vector a pairs with channel e of vector b
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        oa[m] = fma2(ya[m], C[m], mul2(yb[m], NSv[m]));
                        ob[m] = fma2(yb[m], C[m], mul2(ya[m], Sv[m]));
                    }
                } else {
                    // channels (2m, 2m+1) of a vector pair up: pair slot m of
                    // vector a, 4 + m of vector b
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float ca = (m & 1) ? C[m >> 1].y : C[m >> 1].x;
                        const float sa = (m & 1) ? Sv[m >> 1].y : Sv[m >> 1].x;
                        const float cb = (m & 1) ? C[2 + (m >> 1)].y : C[2 + (m >> 1)].x;
                        const float sb = (m & 1) ? Sv[2 + (m >> 1)].y : Sv[2 + (m >> 1)].x;
                        oa[m].x = ya[m].x * ca - ya[m].y * sa;
                        oa[m].y = ya[m].y * ca + ya[m].x * sa;
                        ob[m].x = yb[m].x * cb - yb[m].y * sb;
                        ob[m].y = yb[m].y * cb + yb[m].x * sb;
                    }
                }
                uint8_t* o = (pass == 0 ? qrow : krow) + ooff[k];
                if constexpr (FP8) {
                    const float fa[8] = {oa[0].x, oa[0].y, oa[1].x, oa[1].y,
                                         oa[2].x, oa[2].y, oa[3].x, oa[3].y};
                    const float fb[8] = {ob[0].x, ob[0].y, ob[1].x, ob[1].y,
                                         ob[2].x, ob[2].y, ob[3].x, ob[3].y};
                    st_v2(o, pack8_e4m3_unscaled(fa));
                    st_v2(o + 8 * dv, pack8_e4m3_unscaled(fb));
                } else {
                    st_v4(o, make_uint4(f2_to_bf16x2(oa[0]), f2_to_bf16x2(oa[1]),
                                        f2_to_bf16x2(oa[2]), f2_to_bf16x2(oa[3])));
                    st_v4(o + 16 * dv, make_uint4(f2_to_bf16x2(ob[0]), f2_to_bf16x2(ob[1]),
                                                 f2_to_bf16x2(ob[2]), f2_to_bf16x2(ob[3])));
                }
            }
        }
    }
    if (ctid == 0) {
        if (aborted || *abort_flag) {
            atomicOr(&g_rope3d_status, 1u);
            // Loads of tokens i .. i+stages-1 may still be in flight (each
            // buffer is refilled at its own token's barrier): drain them,
            // bounded.
            for (int64_t j = i; j < n_local && j < i + stages; ++j)
                mbar_wait_bounded(&full[j % stages], (uint32_t)((j / stages) & 1),
                                  a.wait_limit_ns);
        }
        if (v_bulk) bulk_wait_all();
    }
}

// ---------------------------------------------------------------------------
// Fallback kernel: 128-bit loads into registers, no ring.
// ---------------------------------------------------------------------------
template <int D, bool NEOX, bool FP8, int S>
__global__ void __launch_bounds__(kMaxBlock) rope3d_reg_kernel(const Rope3DArgs a) {
    constexpr int L = D / 16;
    constexpr int VPH = D / 8;
    constexpr int HALF = D / 2;
    constexpr int OUTB = FP8 ? 1 : 2;

    extern __shared__ __align__(128) unsigned char smem[];
    float2* cst = reinterpret_cast<float2*>(smem);     // [2][HALF]
    float2* red = cst + 2 * HALF;                      // [2][32]
    uint64_t* gq = reinterpret_cast<uint64_t*>(red + 64);
    float2* tab = reinterpret_cast<float2*>(gq + HALF);

    const int tid = threadIdx.x;
    const int B = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = B >> 5;
    const int l = tid % L;
    const bool norm = a.is_qk_norm != 0;
    const int nq = a.hq * L, nk = a.hk * L, nv = a.hv * VPH;

    setup_angles<D>(a, gq, tab);
    uint4 wqa[S], wqb[S], wka[S], wkb[S];
    load_weights<S>(a, VPH, L, l, tid, B, wqa, wqb, wka, wkb);
    __syncthreads();

    const int64_t row_bytes = (int64_t)(a.hq + a.hk + a.hv) * D * 2;
    const int hw = a.pph * a.ppw;
    const int P = a.ppf * hw;
    const int pstep = (int)((int64_t)gridDim.x % P);
    int s_pos = (int)(((int64_t)blockIdx.x + a.pos_offset) % P);
    const float inv_nq = 1.0f / (float)(a.hq * D > 0 ? a.hq * D : 1);
    const float inv_nk = 1.0f / (float)(a.hk * D > 0 ? a.hk * D : 1);

    int parity = 0;
    for (int64_t t = blockIdx.x; t < a.num_tokens; t += gridDim.x, parity ^= 1) {
        const uint8_t* row = a.qkv + t * row_bytes;
        uint4 qa[S], qb[S], ka[S], kb[S];
#pragma unroll
        for (int k = 0; k < S; ++k) {
            const int slot = tid + k * B;
            const int h = slot / L;
            if (slot < nq) {
                const uint8_t* p = row + (size_t)(h * VPH + l) * 16;
                qa[k] = ld_nc_v4(p); qb[k] = ld_nc_v4(p + L * 16);
            }
            if (slot < nk) {
                const uint8_t* p = row + (size_t)((a.hq + h) * VPH + l) * 16;
                ka[k] = ld_nc_v4(p); kb[k] = ld_nc_v4(p + L * 16);
            }
        }
        const uint8_t* vrow = row + (size_t)(a.hq + a.hk) * VPH * 16;
        uint8_t* vout = a.v_out + t * (int64_t)nv * 8 * OUTB;
        for (int vi = tid; vi < nv; vi += B) {
            const uint4 v = ld_nc_v4(vrow + (size_t)vi * 16);
            if constexpr (FP8) {
                float f[8];
                unpack8(v, f);
                st_v2(vout + (size_t)vi * 8, pack8_e4m3(f, a.v_scale));
            } else {
                st_v4(vout + (size_t)vi * 16, v);
            }
        }
        {
            const int pf = s_pos / hw;
            const int rem = s_pos - pf * hw;
            const int ph = rem / a.ppw;
            const int pw = rem - ph * a.ppw;
            for (int j = tid; j < HALF; j += B)
                cst[parity * HALF + j] = pair_cos_sin(a, gq, tab, j, pf, ph, pw);
        }
        s_pos += pstep;
        if (s_pos >= P) s_pos -= P;
        if (norm) {
            float2 sq2 = make_float2(0.0f, 0.0f), sk2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int k = 0; k < S; ++k) {
                const int slot = tid + k * B;
                if (slot < nq) sq2 = ssq_pair(qa[k], qb[k], sq2);
                if (slot < nk) sk2 = ssq_pair(ka[k], kb[k], sk2);
            }
            const float sq = warp_sum(sq2.x + sq2.y);
            const float sk = warp_sum(sk2.x + sk2.y);
            if (lane == 0) red[parity * 32 + warp] = make_float2(sq, sk);
        }
        __syncthreads();
        float rq = 1.0f, rk = 1.0f;
        if (norm) {
            float tq = 0.0f, tk = 0.0f;
            for (int w = 0; w < nwarps; ++w) {
                const float2 v = red[parity * 32 + w];
                tq += v.x; tk += v.y;
            }
            rq = rsqrtf(tq * inv_nq + a.eps);
            rk = rsqrtf(tk * inv_nk + a.eps);
        }
        float cs[8], sn[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float2 v = cst[parity * HALF + slot_of<D, NEOX>(l, k)];
            cs[k] = v.x; sn[k] = v.y;
        }
#pragma unroll
        for (int k = 0; k < S; ++k) {
            const int slot = tid + k * B;
            const int h = slot / L;
            if (slot < nq)
                apply_slot<D, NEOX, FP8>(qa[k], qb[k], wqa[k], wqb[k], norm, rq, cs, sn,
                                         a.q_out + (t * a.hq + h) * D * OUTB, l, a.q_scale);
            if (slot < nk)
                apply_slot<D, NEOX, FP8>(ka[k], kb[k], wka[k], wkb[k], norm, rk, cs, sn,
                                         a.k_out + (t * a.hk + h) * D * OUTB, l, a.q_scale);
        }
    }
}

// Launch with programmatic stream serialisation: the kernel may start its
// prologue while the previous kernel on the stream finishes (the kernel waits
// with griddepcontrol.wait before it touches global memory).
template <typename K, typename A>
cudaError_t launch_overlapped(K kern, int grid, int block, int smem, cudaStream_t stream,
                              const A& args) {
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

int device_sms() {
    int sms = 0;
    return cached_sm_count(&sms) == cudaSuccess ? sms : 0;
}

// Whether a CTA builds the shared cos/sin table: it must fit, and its
// entries (one sincos each, per CTA) must not outnumber the angles the CTA
// would otherwise evaluate per token (half a head's channels for each of its
// tokens). Short calls (a few thousand tokens over all SMs) evaluate them
// per token instead.
bool table_pays(const Rope3DArgs& a, int half) {
    if ((int64_t)a.table_entries * 8 > kMaxTableBytes) return false;
    const int sms = std::max(1, device_sms());
    const int64_t tokens_per_cta = (a.num_tokens + sms - 1) / sms;
    return (int64_t)a.table_entries <= tokens_per_cta * half;
}

template <typename K>
cudaError_t launch_grid(K kern, int block, int smem, int64_t tokens, const Rope3DArgs& args,
                        cudaStream_t stream, int* grid_out) {
    int per_sm = 0;
    cudaError_t e =
        cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block, smem, &per_sm);
    if (e != cudaSuccess) return e;
    const int sms = device_sms();
    if (sms <= 0) return cudaErrorNoDevice;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int grid = (int)std::min<int64_t>((int64_t)sms * per_sm, tokens);
    kern<<<grid, block, smem, stream>>>(args);
    *grid_out = grid;
    return cudaGetLastError();
}

// S: the Q slot and K slot pairs per thread at block_reg threads (the
// fallback kernel, and the pipelined kernel when Q and K have as many heads).
// With unequal head counts the pipelined kernel instead deals 2S slots per
// thread from the list [Q slots | K slots] over block_mg threads, so that every
// thread still has the same work.
template <int D, bool NEOX, bool FP8, int S>
cudaError_t run(const Rope3DArgs& a, int block_mg, int block_reg, cudaStream_t stream,
                LaunchInfo* info) {
    constexpr int HALF = D / 2;
    const bool mixed = a.hq != a.hk;
    int block = mixed ? block_mg : block_reg;
    Rope3DArgs args = a;
    const bool partial = a.mode == kModePartialSsq;
    const int table_bytes = a.table_entries * 8;
    args.use_table = (!partial && table_pays(a, HALF)) ? 1 : 0;
    const int used_table = args.use_table ? table_bytes : 0;
    const int row_bytes = partial ? (a.hq + a.hk) * D * 2 : (a.hq + a.hk + a.hv) * D * 2;
    const int weight_floats = (a.is_qk_norm && !partial) ? (a.hq + a.hk) * D : 0;
    if (args.norm_q_elems == 0) args.norm_q_elems = a.hq * D;
    if (args.norm_k_elems == 0) args.norm_k_elems = a.hk * D;
    // Pipelines per CTA: as many groups as fit in 24 warps and in shared memory,
    // each with a ring of 3 row buffers (2 if 3 do not fit even for one group).
    const int warps = block / 32;
    int groups = std::max(1, std::min(kMaxGroups, 24 / warps));
    int stages = 0;
    for (; groups >= 1; --groups) {
        for (stages = 3; stages >= 2; --stages) {
            if (mg_layout(D, groups, stages, row_bytes, weight_floats, used_table).total <=
                kSmemPerSm - 1024)
                break;
        }
        if (stages >= 2) break;
    }
    // Do not start more pipelines than there are tokens.
    const int sms = device_sms();
    if (sms <= 0) return cudaErrorNoDevice;
    while (groups > 1 && (int64_t)sms * (groups - 1) >= a.num_tokens) --groups;
    int grid = 0, smem = 0, id = 0;
    cudaError_t e;
    if (groups >= 1 && stages >= 2) {
        args.stages = stages;
        args.groups = groups;
        args.v_bulk = FP8 ? 0 : 1;
        if (args.wait_limit_ns == 0) args.wait_limit_ns = 2000000000ull;  // 2 s
        smem = mg_layout(D, groups, stages, row_bytes, weight_floats, used_table).total;
        void (*kern)(const Rope3DArgs) = mixed ? rope3d_mg_kernel<D, NEOX, FP8, 2 * S, true>
                                               : rope3d_mg_kernel<D, NEOX, FP8, S, false>;
        int per_sm = 0;
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block * groups, smem,
                                      &per_sm);
        if (e == cudaSuccess && per_sm < 1) e = cudaErrorInvalidConfiguration;
        if (e == cudaSuccess) {
            grid = (int)std::min<int64_t>(sms, (a.num_tokens + groups - 1) / groups);
            e = launch_overlapped(kern, grid, block * groups, smem, stream, args);
            if (e != cudaSuccess) {
                cudaGetLastError();
                forget_kernel(reinterpret_cast<const void*>(kern));
                e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block * groups,
                                              smem, &per_sm);
                if (e == cudaSuccess) e = launch_overlapped(kern, grid, block * groups, smem, stream, args);
            }
        }
        id = 3100;
        block *= groups;
    } else if (a.mode != kModeWhole) {
        return cudaErrorNotSupported;  // the tensor-parallel passes run on the pipelined kernel
    } else {
        smem = 2 * HALF * 8 + 64 * 8 + HALF * 8 + used_table;
        block = block_reg;
        e = launch_grid(rope3d_reg_kernel<D, NEOX, FP8, S>, block, smem, a.num_tokens, args,
                        stream, &grid);
        id = 3000;
    }
    if (info) {
        info->grid = grid;
        info->block = block;
        info->smem = smem;
        info->kernel_id = id + D / 64 * 10 + (NEOX ? 4 : 0) + (FP8 ? 2 : 0) + (S > 1);
    }
    return e;
}

// The register-resident kernel for a whole-transform call, when its shape
// fits: NS slots per thread, at most rr_max_threads<NS>() threads per CTA, a
// two-buffer ring per pipeline in shared memory. Returns cudaErrorNotSupported
// (nothing launched) otherwise.
template <int D, bool NEOX, bool FP8, int NS>
cudaError_t run_rr(const Rope3DArgs& a, cudaStream_t stream, LaunchInfo* info) {
    constexpr int L = D / 16;
    if (a.mode == kModePartialSsq) return cudaErrorNotSupported;
    const bool mixed = a.hq != a.hk;
    const int nq = a.hq * L, nk = a.hk * L;
    const int need = mixed ? (nq + nk + NS - 1) / NS : (std::max(nq, nk) + NS / 2 - 1) / (NS / 2);
    int bg = std::max(32, (need + 31) / 32 * 32);
    const int max_threads = rr_max_threads<NS>();
    if (bg > max_threads) return cudaErrorNotSupported;
    Rope3DArgs args = a;
    const int table_bytes = a.table_entries * 8;
    args.use_table = table_pays(a, D / 2) ? 1 : 0;
    const int used_table = args.use_table ? table_bytes : 0;
    const int row_bytes = (a.hq + a.hk + a.hv) * D * 2;
    const bool bw = !mixed;  // the kernel's BW: bf16 weights in shared memory
    const int weight_floats = a.is_qk_norm ? (a.hq + a.hk) * D / (bw ? 2 : 1) : 0;
    if (args.norm_q_elems == 0) args.norm_q_elems = a.hq * D;
    if (args.norm_k_elems == 0) args.norm_k_elems = a.hk * D;
    int groups = std::min(kMaxGroups, max_threads / bg);
    const int sms = device_sms();
    if (sms <= 0) return cudaErrorNoDevice;
    while (groups > 1 && (int64_t)sms * (groups - 1) >= a.num_tokens) --groups;
    for (; groups >= 1; --groups)
        if (mg_layout(D, groups, 2, row_bytes, weight_floats, used_table).total <= kSmemPerSm - 1024)
            break;
    if (groups < 1) return cudaErrorNotSupported;
    int stages = 2;
    if (mg_layout(D, groups, 3, row_bytes, weight_floats, used_table).total <= kSmemPerSm - 1024)
        stages = 3;
    args.stages = stages;
    args.groups = groups;
    args.v_bulk = FP8 ? 0 : 1;
    if (args.wait_limit_ns == 0) args.wait_limit_ns = 2000000000ull;  // 2 s
    const int smem = mg_layout(D, groups, stages, row_bytes, weight_floats, used_table).total;
    const int block = bg * groups;
    void (*kern)(const Rope3DArgs) = mixed ? rope3d_rr_kernel<D, NEOX, FP8, NS, true>
                                           : rope3d_rr_kernel<D, NEOX, FP8, NS, false>;
    int per_sm = 0;
    cudaError_t e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block, smem,
                                              &per_sm);
    if (e == cudaSuccess && per_sm < 1) e = cudaErrorInvalidConfiguration;
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(sms, (a.num_tokens + groups - 1) / groups);
    e = launch_overlapped(kern, grid, block, smem, stream, args);
    if (e != cudaSuccess) {
        cudaGetLastError();
        forget_kernel(reinterpret_cast<const void*>(kern));
        e = cached_smem_and_occupancy(reinterpret_cast<const void*>(kern), block, smem, &per_sm);
        if (e == cudaSuccess) e = launch_overlapped(kern, grid, block, smem, stream, args);
    }
    if (info) {
        info->grid = grid;
        info->block = block;
        info->smem = smem;
        info->kernel_id = 3200 + D / 64 * 10 + (NEOX ? 4 : 0) + (FP8 ? 2 : 0) + (mixed ? 1 : 0);
    }
    return e;
}

template <int D, bool NEOX, bool FP8>
cudaError_t run_s(const Rope3DArgs& a, cudaStream_t stream, LaunchInfo* info) {
    constexpr int L = D / 16;
    // The register-resident kernel where it measured faster (NeoX pairs or
    // grouped-query heads with the norm), and for the per-axis NeoX layout,
    // which only it builds; the pipelined kernel for the rest.
    if (a.mode != kModePartialSsq &&
        (a.neox_per_axis || (a.is_qk_norm && (NEOX || a.hq != a.hk)))) {
        const cudaError_t e = run_rr<D, NEOX, FP8, 4>(a, stream, info);
        if (e != cudaErrorNotSupported || a.neox_per_axis) return e;
    }
    const int slots = std::max(std::max(a.hq, a.hk), 1) * L;
    int S = (slots + kMaxBlock - 1) / kMaxBlock;
    if (S > 4) return cudaErrorInvalidValue;  // rejected earlier by the host checks
    S = S <= 1 ? 1 : (S <= 2 ? 2 : 4);
    int block_reg = ((slots + S - 1) / S + 31) / 32 * 32;
    const int all_slots = std::max(a.hq + a.hk, 1) * L;
    int block_mg = ((all_slots + 2 * S - 1) / (2 * S) + 31) / 32 * 32;
    // With few Q/K heads, widen the block so that V and the per-token cos/sin
    // have enough threads.
    const int v_vectors = a.hv * (D / 8);
    for (int* b : {&block_reg, &block_mg})
        while (*b < 256 && (*b < v_vectors / 2 || *b < D / 2)) *b += 32;
    switch (S) {
        case 1: return run<D, NEOX, FP8, 1>(a, block_mg, block_reg, stream, info);
        case 2: return run<D, NEOX, FP8, 2>(a, block_mg, block_reg, stream, info);
        default: return run<D, NEOX, FP8, 4>(a, block_mg, block_reg, stream, info);
    }
}

template <int D>
cudaError_t run_d(const Rope3DArgs& a, int neox, int fp8, cudaStream_t stream,
                  LaunchInfo* info) {
    if (neox) {
        return fp8 ? run_s<D, true, true>(a, stream, info) : run_s<D, true, false>(a, stream, info);
    }
    return fp8 ? run_s<D, false, true>(a, stream, info) : run_s<D, false, false>(a, stream, info);
}

}  // namespace

cudaError_t launch_rope3d(const Rope3DArgs& a, int head_dim, int neox, int fp8,
                          cudaStream_t stream, LaunchInfo* info) {
    switch (head_dim) {
        case 64: return run_d<64>(a, neox, fp8, stream, info);
        case 128: return run_d<128>(a, neox, fp8, stream, info);
        case 256: return run_d<256>(a, neox, fp8, stream, info);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t read_device_status(uint32_t* out, int clear, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_rope3d_status, sizeof(uint32_t), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && clear) {
        const uint32_t zero = 0;
        e = cudaMemcpyToSymbolAsync(g_rope3d_status, &zero, sizeof(uint32_t), 0,
                                    cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    }
    return e;
}

// Largest number of Q or K heads the 3D kernels take for a head size
// (S <= 4 slots per thread at 512 threads).
int rope3d_max_heads(int head_dim) { return 4 * kMaxBlock / (head_dim / 16); }

}  // namespace qknr
