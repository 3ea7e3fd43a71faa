// Packed-QKV across-heads RMSNorm + 3D RoPE + V copy (+ FP8 E4M3 output).
//
// Computes the operation of "flashinfer.norm.fused_qk_rmsnorm_rope" (FlashInfer
// API docs; summary, Parameters, Returns) in one pass over HBM: every input
// byte is read once with 128-bit loads, every output byte written once with
// 128-bit (bf16) or 64-bit (E4M3) stores, and nothing else touches memory.
//
// Layout of the work. A CTA is persistent and walks tokens t = blockIdx.x,
// blockIdx.x + gridDim.x, ... For one token the CTA holds the whole Q and K
// part of the row in registers: thread tid owns, for S "slots" (head, l),
// the two 16-byte vectors l and l + D/16 of that head (l = tid mod D/16, the
// same for every slot of the thread). Vector l's channel e pairs with vector
// l + D/16's channel e in NeoX mode; in interleaved mode each vector's
// adjacent channels pair up. Either way a thread's 8 rotation pairs sit at
// fixed pair slots, so their frequencies, weights and table columns are set up
// once per CTA. V vectors are streamed straight to v_out.
//
// Per token: issue every load, store V, reduce sum(x^2) of Q and of K over the
// CTA (warp shuffles, one shared-memory exchange, one barrier), then scale,
// rotate, convert and store. cos/sin come from a per-CTA shared-memory table
// of every (axis, position, frequency) triple -- at most ppf*Cf/2 + pph*Ch/2 +
// ppw*Cw/2 entries -- built once per CTA with an exact fixed-point angle, or,
// when the table would not fit, from the same angle computed per token.
#include "common.cuh"
#include "launch.h"

#include <algorithm>

namespace qknr {

namespace {

constexpr int kMaxBlock = 512;
constexpr int kMaxTableBytes = 64 * 1024;

template <int D, bool NEOX, bool FP8, int S>
__global__ void __launch_bounds__(kMaxBlock) rope3d_kernel(const Rope3DArgs a) {
    constexpr int L = D / 16;   // threads per head
    constexpr int VPH = D / 8;  // 16-byte vectors per head
    constexpr int HALF = D / 2;
    constexpr int SV = 2 * S;  // V vectors per thread issued with the Q/K loads
    constexpr int OUTB = FP8 ? 1 : 2;

    extern __shared__ __align__(16) unsigned char smem[];
    uint64_t* gq = reinterpret_cast<uint64_t*>(smem);                  // [HALF]
    float2* red = reinterpret_cast<float2*>(smem + HALF * 8);         // [2][32]
    float2* tab = reinterpret_cast<float2*>(smem + HALF * 8 + 512);  // [table_entries]

    const int tid = threadIdx.x;
    const int B = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = B >> 5;
    const int l = tid % L;
    const int hcf = a.cf >> 1, hch = a.ch >> 1, hcw = a.cw >> 1;
    const bool norm = a.is_qk_norm != 0;

    // Frequencies of the HALF pair slots, as 64-bit fractions of a turn.
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
    const int nf = a.ppf * hcf, nh = a.pph * hch;
    if (a.use_table) {
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
        __syncthreads();
    }

    // This thread's 8 pair slots: axis and index inside the axis group.
    int pax[8], pcol[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int j = NEOX ? 8 * l + k : (k < 4 ? 4 * l + k : 4 * (l + L) + (k - 4));
        if (j < hcf) {
            pax[k] = 0; pcol[k] = j;
        } else if (j < hcf + hch) {
            pax[k] = 1; pcol[k] = j - hcf;
        } else {
            pax[k] = 2; pcol[k] = j - hcf - hch;
        }
    }

    const int nq = a.hq * L, nk = a.hk * L, nv = a.hv * VPH;
    // Weights of this thread's slots stay in registers for the whole kernel.
    uint4 wqa[S], wqb[S], wka[S], wkb[S];
#pragma unroll
    for (int i = 0; i < S; ++i) {
        const int slot = tid + i * B;
        const uint4 one = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        wqa[i] = wqb[i] = wka[i] = wkb[i] = one;
        if (norm && slot < nq) {
            const int h = slot / L;
            const uint4* w = reinterpret_cast<const uint4*>(a.q_weight) + h * VPH + l;
            wqa[i] = w[0]; wqb[i] = w[L];
        }
        if (norm && slot < nk) {
            const int h = slot / L;
            const uint4* w = reinterpret_cast<const uint4*>(a.k_weight) + h * VPH + l;
            wka[i] = w[0]; wkb[i] = w[L];
        }
    }

    const int64_t row_bytes = (int64_t)(a.hq + a.hk + a.hv) * D * 2;
    const int hw = a.pph * a.ppw;
    const int64_t P = (int64_t)a.ppf * hw;
    const float inv_nq = 1.0f / (float)(a.hq * D > 0 ? a.hq * D : 1);
    const float inv_nk = 1.0f / (float)(a.hk * D > 0 ? a.hk * D : 1);

    int parity = 0;
    for (int64_t t = blockIdx.x; t < a.num_tokens; t += gridDim.x, parity ^= 1) {
        const uint8_t* row = a.qkv + t * row_bytes;
        uint4 qa[S], qb[S], ka[S], kb[S], vv[SV];
#pragma unroll
        for (int i = 0; i < S; ++i) {
            const int slot = tid + i * B;
            const int h = slot / L;
            if (slot < nq) {
                const uint8_t* p = row + (size_t)(h * VPH + l) * 16;
                qa[i] = ld_nc_v4(p); qb[i] = ld_nc_v4(p + L * 16);
            }
            if (slot < nk) {
                const uint8_t* p = row + (size_t)((a.hq + h) * VPH + l) * 16;
                ka[i] = ld_nc_v4(p); kb[i] = ld_nc_v4(p + L * 16);
            }
        }
        const uint8_t* vrow = row + (size_t)(a.hq + a.hk) * VPH * 16;
#pragma unroll
        for (int i = 0; i < SV; ++i) {
            const int vi = tid + i * B;
            if (vi < nv) vv[i] = ld_nc_v4(vrow + (size_t)vi * 16);
        }

        // Patch coordinates of this token.
        const int64_t s64 = (t + a.pos_offset) % P;
        const int s = (int)s64;
        const int pf = s / hw;
        const int rem = s - pf * hw;
        const int ph = rem / a.ppw;
        const int pw = rem - ph * a.ppw;

        // V: bit copy (bf16) or E4M3(v * v_scale).
        uint8_t* vout = a.v_out + t * (int64_t)nv * 8 * OUTB;
#pragma unroll
        for (int i = 0; i < SV; ++i) {
            const int vi = tid + i * B;
            if (vi < nv) {
                if constexpr (FP8) {
                    float f[8];
                    unpack8(vv[i], f);
                    st_v2(vout + (size_t)vi * 8, pack8_e4m3(f, a.v_scale));
                } else {
                    st_v4(vout + (size_t)vi * 16, vv[i]);
                }
            }
        }
        for (int vi = tid + SV * B; vi < nv; vi += B) {  // heads beyond the up-front batch
            const uint4 v = ld_nc_v4(vrow + (size_t)vi * 16);
            if constexpr (FP8) {
                float f[8];
                unpack8(v, f);
                st_v2(vout + (size_t)vi * 8, pack8_e4m3(f, a.v_scale));
            } else {
                st_v4(vout + (size_t)vi * 16, v);
            }
        }

        // Across-heads RMS of Q and of K.
        float rq = 1.0f, rk = 1.0f;
        if (norm) {
            float sq = 0.0f, sk = 0.0f;
#pragma unroll
            for (int i = 0; i < S; ++i) {
                const int slot = tid + i * B;
                if (slot < nq) {
                    float fa[8], fb[8];
                    unpack8(qa[i], fa); unpack8(qb[i], fb);
#pragma unroll
                    for (int e = 0; e < 8; ++e) sq += fa[e] * fa[e] + fb[e] * fb[e];
                }
                if (slot < nk) {
                    float fa[8], fb[8];
                    unpack8(ka[i], fa); unpack8(kb[i], fb);
#pragma unroll
                    for (int e = 0; e < 8; ++e) sk += fa[e] * fa[e] + fb[e] * fb[e];
                }
            }
            sq = warp_sum(sq);
            sk = warp_sum(sk);
            float2* rb = red + parity * 32;
            if (lane == 0) rb[warp] = make_float2(sq, sk);
            __syncthreads();
            float tq = 0.0f, tk = 0.0f;
            for (int w = 0; w < nwarps; ++w) {
                const float2 v = rb[w];
                tq += v.x; tk += v.y;
            }
            rq = rsqrtf(tq * inv_nq + a.eps);
            rk = rsqrtf(tk * inv_nk + a.eps);
        }

        // cos/sin of this thread's 8 pairs.
        float cs[8], sn[8];
        if (a.use_table) {
            const int r0 = pf * hcf, r1 = nf + ph * hch, r2 = nf + nh + pw * hcw;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int base = pax[k] == 0 ? r0 : (pax[k] == 1 ? r1 : r2);
                const float2 v = tab[base + pcol[k]];
                cs[k] = v.x; sn[k] = v.y;
            }
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int j = NEOX ? 8 * l + k : (k < 4 ? 4 * l + k : 4 * (l + L) + (k - 4));
                const int pos = pax[k] == 0 ? pf : (pax[k] == 1 ? ph : pw);
                turn_sincos((uint32_t)pos, gq[j], &sn[k], &cs[k]);
            }
        }

        // Scale, rotate, convert, store: Q then K.
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int nslot = part ? nk : nq;
            const float r = part ? rk : rq;
            const int H = part ? a.hk : a.hq;
            uint8_t* out = (part ? a.k_out : a.q_out) + t * (int64_t)H * D * OUTB;
            const float scale = a.q_scale;
#pragma unroll
            for (int i = 0; i < S; ++i) {
                const int slot = tid + i * B;
                if (slot >= nslot) continue;
                const int h = slot / L;
                float xa[8], xb[8];
                unpack8(part ? ka[i] : qa[i], xa);
                unpack8(part ? kb[i] : qb[i], xb);
                if (norm) {
                    float wa[8], wb[8];
                    unpack8(part ? wka[i] : wqa[i], wa);
                    unpack8(part ? wkb[i] : wqb[i], wb);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        xa[e] = xa[e] * r * wa[e];
                        xb[e] = xb[e] * r * wb[e];
                    }
                }
                float oa[8], ob[8];
                if constexpr (NEOX) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        oa[e] = xa[e] * cs[e] - xb[e] * sn[e];
                        ob[e] = xb[e] * cs[e] + xa[e] * sn[e];
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        oa[2 * m] = xa[2 * m] * cs[m] - xa[2 * m + 1] * sn[m];
                        oa[2 * m + 1] = xa[2 * m + 1] * cs[m] + xa[2 * m] * sn[m];
                        ob[2 * m] = xb[2 * m] * cs[4 + m] - xb[2 * m + 1] * sn[4 + m];
                        ob[2 * m + 1] = xb[2 * m + 1] * cs[4 + m] + xb[2 * m] * sn[4 + m];
                    }
                }
                if constexpr (FP8) {
                    uint8_t* p = out + (size_t)h * D + 8 * l;
                    st_v2(p, pack8_e4m3(oa, scale));
                    st_v2(p + 8 * L, pack8_e4m3(ob, scale));
                } else {
                    uint8_t* p = out + (size_t)(h * VPH + l) * 16;
                    st_v4(p, pack8_bf16(oa));
                    st_v4(p + 16 * L, pack8_bf16(ob));
                }
            }
        }
    }
}

template <int D, bool NEOX, bool FP8, int S>
cudaError_t run(const Rope3DArgs& a, int block, cudaStream_t stream, LaunchInfo* info) {
    auto kern = rope3d_kernel<D, NEOX, FP8, S>;
    Rope3DArgs args = a;
    const int fixed = (D / 2) * 8 + 512;
    const int table_bytes = a.table_entries * 8;
    args.use_table = table_bytes <= kMaxTableBytes ? 1 : 0;
    const int smem = fixed + (args.use_table ? table_bytes : 0);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             smem);
        if (e != cudaSuccess) return e;
    }
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, block,
                                                                            smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const int64_t want = (int64_t)sms * per_sm;
    const int grid = (int)std::min<int64_t>(want, a.num_tokens);
    kern<<<grid, block, smem, stream>>>(args);
    if (info) {
        info->grid = grid;
        info->block = block;
        info->smem = smem;
        info->kernel_id = 3000 + D * 10 + (NEOX ? 1 : 0) * 4 + (FP8 ? 2 : 0) + (S > 1);
    }
    return cudaGetLastError();
}

template <int D, bool NEOX, bool FP8>
cudaError_t run_s(const Rope3DArgs& a, cudaStream_t stream, LaunchInfo* info) {
    constexpr int L = D / 16;
    int slots = std::max(std::max(a.hq, a.hk), 1) * L;
    const int v_vectors = a.hv * (D / 8);
    int S = (slots + kMaxBlock - 1) / kMaxBlock;
    if (S > 4) return cudaErrorInvalidValue;  // rejected earlier by the host checks
    S = S <= 1 ? 1 : (S <= 2 ? 2 : 4);
    int block = ((slots + S - 1) / S + 31) / 32 * 32;
    // With few Q/K heads, widen the block to cover V in the up-front batch.
    while (block < kMaxBlock && 2 * S * block < v_vectors && block < 256) block += 32;
    switch (S) {
        case 1: return run<D, NEOX, FP8, 1>(a, block, stream, info);
        case 2: return run<D, NEOX, FP8, 2>(a, block, stream, info);
        default: return run<D, NEOX, FP8, 4>(a, block, stream, info);
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

// Largest number of Q or K heads the 3D kernel takes for a head size
// (S <= 4 slots per thread at 512 threads).
int rope3d_max_heads(int head_dim) { return 4 * kMaxBlock / (head_dim / 16); }

}  // namespace qknr
