// C ABI of libqknr.so (declared in include/qknr.h): argument checks, pointer
// classification, and dispatch to the kernel launchers. Nothing here
// allocates, synchronises or touches the data.
#include "qknr.h"

#include "launch.h"
#include "ucpe_launch.h"

#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>

namespace {

thread_local char g_detail[320] = "";

// Timeout-path test hook (qknr_test_set_wait_fault).
std::atomic<uint32_t> g_fault_extra_bytes{0};
std::atomic<uint64_t> g_fault_limit_ns{0};

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
    return code;
}

int ok() {
    g_detail[0] = '\0';
    return QKNR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A pointer the current device can dereference: its own device memory,
// managed memory, or host memory registered with CUDA (page-locked). On
// success *dev_ptr is the address a kernel must use.
int classify(const void* p, const char* name, int device, const void** dev_ptr) {
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(QKNR_ERR_POINTER, "%s: cudaPointerGetAttributes failed (%s)", name,
                    cudaGetErrorString(e));
    }
    switch (attr.type) {
        case cudaMemoryTypeDevice:
            if (attr.device != device)
                return fail(QKNR_ERR_POINTER, "%s: memory of device %d, current device is %d",
                            name, attr.device, device);
            *dev_ptr = p;
            return QKNR_OK;
        case cudaMemoryTypeManaged:
            *dev_ptr = p;
            return QKNR_OK;
        case cudaMemoryTypeHost:
            if (attr.devicePointer == nullptr)
                return fail(QKNR_ERR_POINTER, "%s: host memory not mapped for the device", name);
            *dev_ptr = attr.devicePointer;
            return QKNR_OK;
        default:
            return fail(QKNR_ERR_POINTER,
                        "%s: not memory the device can access (pageable host memory?)", name);
    }
}

// A [rows, row_bytes] byte region whose rows start stride_bytes apart.
struct Span {
    const void* p;
    uint64_t bytes;  // total extent, first byte to last
    int64_t row_bytes = 0;
    int64_t stride_bytes = 0;
};

// Bytes spanned by a [rows, cols] tensor of `elem` bytes with a row stride of
// `stride` elements.
uint64_t span_bytes(int64_t rows, int64_t cols, int64_t stride, int elem) {
    if (rows <= 0 || cols <= 0) return 0;
    return (uint64_t)((rows - 1) * stride + cols) * (uint64_t)elem;
}

Span rows_span(const void* p, int64_t rows, int64_t cols, int64_t stride, int elem) {
    Span s{p, span_bytes(rows, cols, stride, elem)};
    s.row_bytes = cols * elem;
    s.stride_bytes = stride * elem;
    return s;
}

// Whether two regions share a byte. Two row sets with the same row stride
// whose rows interleave without touching (q and k heads inside one packed QKV
// buffer) do not overlap; other cases fall back to comparing extents.
bool overlap(Span a, Span b) {
    if (a.p == nullptr || b.p == nullptr || a.bytes == 0 || b.bytes == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    if (!(a0 < b0 + b.bytes && b0 < a0 + a.bytes)) return false;
    const int64_t s = a.stride_bytes;
    if (s > 0 && s == b.stride_bytes && a.row_bytes <= s && b.row_bytes <= s) {
        const int64_t d = (int64_t)(b0 - a0);
        const int64_t m = ((d % s) + s) % s;  // where b's rows start inside a's period
        if (m >= a.row_bytes && m + b.row_bytes <= s) return false;
    }
    return true;
}

int cuda_fail(cudaError_t e, const char* what) {
    cudaGetLastError();
    return fail(QKNR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

namespace qknr {
int rope3d_max_heads(int head_dim);
}

extern "C" {

int qknr_abi_version(void) { return QKNR_ABI_VERSION; }

const char* qknr_status_string(int status) {
    switch (status) {
        case QKNR_OK: return "ok";
        case QKNR_ERR_NULL: return "a required pointer is NULL";
        case QKNR_ERR_SHAPE: return "sizes or parameters break the contract";
        case QKNR_ERR_UNSUPPORTED: return "not supported by this library";
        case QKNR_ERR_ALIGN: return "a pointer or stride is not 16-byte aligned";
        case QKNR_ERR_ALIAS: return "an output overlaps an input";
        case QKNR_ERR_POINTER: return "a pointer the current device cannot access";
        case QKNR_ERR_CUDA: return "CUDA runtime error";
        default: return "unknown status";
    }
}

const char* qknr_last_error_detail(void) { return g_detail; }

int qknr_test_set_wait_fault(uint32_t extra_bytes, uint64_t limit_ns) {
    if (extra_bytes != 0 && (extra_bytes % 16 != 0 || limit_ns == 0))
        return fail(QKNR_ERR_SHAPE, "extra_bytes must be a multiple of 16 and limit_ns > 0");
    g_fault_limit_ns.store(limit_ns);
    g_fault_extra_bytes.store(extra_bytes);
    return ok();
}

int qknr_device_status(void* cuda_stream, uint32_t* status_out, int32_t clear) {
    if (!status_out) return fail(QKNR_ERR_NULL, "status_out is NULL");
    uint32_t v = 0, w = 0;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    uint32_t u = 0;
    cudaError_t e = qknr::read_device_status(&v, clear, st);
    if (e == cudaSuccess) e = qknr::read_table_status(&w, clear, st);
    if (e == cudaSuccess) e = qknr::read_ucpe_status(&u, clear, st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    *status_out = v | w | u;
    return ok();
}

int qknr_rope_table(const void* q, const void* k, void* q_out, void* k_out,
                    const void* q_weight, const void* k_weight, const void* rope_table,
                    int32_t table_dtype, int32_t act_dtype, int64_t num_tokens, int32_t heads_q,
                    int32_t heads_k, int32_t head_dim, int32_t rotary_dim, int64_t q_token_stride,
                    int64_t k_token_stride, int64_t q_out_token_stride,
                    int64_t k_out_token_stride, float eps, int32_t interleaved,
                    void* cuda_stream) {
    // ---- shape checks (host only) ----
    if (num_tokens < 0) return fail(QKNR_ERR_SHAPE, "num_tokens < 0");
    if (heads_q < 0 || heads_k < 0) return fail(QKNR_ERR_SHAPE, "negative head count");
    if (head_dim < 1 || head_dim > 256)
        return fail(QKNR_ERR_SHAPE, "head_dim %d outside 1..256", head_dim);
    const int32_t R = rotary_dim == 0 ? head_dim : rotary_dim;
    if (R < 2 || (R & 1) || R > head_dim)
        return fail(QKNR_ERR_SHAPE, "rotary_dim %d must be even and <= head_dim %d", R,
                    head_dim);
    if (act_dtype != QKNR_DT_BF16 && act_dtype != QKNR_DT_F16)
        return fail(QKNR_ERR_SHAPE, "activation dtype must be bfloat16 or float16");
    if (table_dtype != QKNR_DT_F32 && table_dtype != act_dtype)
        return fail(QKNR_ERR_SHAPE, "rope_table dtype must be float32 or the activation dtype");
    if (!(eps >= 0.0f) || std::isinf(eps)) return fail(QKNR_ERR_SHAPE, "eps must be >= 0");
    const int64_t qrow = (int64_t)heads_q * head_dim, krow = (int64_t)heads_k * head_dim;
    const int64_t qs = q_token_stride ? q_token_stride : qrow;
    const int64_t ks = k_token_stride ? k_token_stride : krow;
    const int64_t qos = q_out_token_stride ? q_out_token_stride : qrow;
    const int64_t kos = k_out_token_stride ? k_out_token_stride : krow;
    if (qs < qrow || ks < krow || qos < qrow || kos < krow)
        return fail(QKNR_ERR_SHAPE, "a token stride is smaller than heads*head_dim");
    if (num_tokens == 0 || (heads_q == 0 && heads_k == 0)) return ok();

    // ---- pointers ----
    const bool has_q = heads_q > 0, has_k = heads_k > 0;
    if (!rope_table) return fail(QKNR_ERR_NULL, "rope_table is NULL");
    if (has_q && (!q || !q_out || !q_weight)) return fail(QKNR_ERR_NULL, "q, q_out or q_weight is NULL");
    if (has_k && (!k || !k_out || !k_weight)) return fail(QKNR_ERR_NULL, "k, k_out or k_weight is NULL");
    const int tb = table_dtype == QKNR_DT_F32 ? 4 : 2;
    const Span sq = rows_span(q, num_tokens, qrow, qs, 2);
    const Span sk = rows_span(k, num_tokens, krow, ks, 2);
    const Span sqo = rows_span(q_out, num_tokens, qrow, qos, 2);
    const Span sko = rows_span(k_out, num_tokens, krow, kos, 2);
    const Span stab{rope_table, (uint64_t)num_tokens * R * tb};
    const bool q_inplace = has_q && q_out == q;
    const bool k_inplace = has_k && k_out == k;
    if (q_inplace && qos != qs) return fail(QKNR_ERR_ALIAS, "in-place q needs the same stride");
    if (k_inplace && kos != ks) return fail(QKNR_ERR_ALIAS, "in-place k needs the same stride");
    if (has_q) {
        if (!q_inplace && overlap(sqo, sq)) return fail(QKNR_ERR_ALIAS, "q_out overlaps q");
        if (has_k && overlap(sqo, sk)) return fail(QKNR_ERR_ALIAS, "q_out overlaps k");
        if (overlap(sqo, stab)) return fail(QKNR_ERR_ALIAS, "q_out overlaps rope_table");
        if (overlap(sqo, Span{q_weight, (uint64_t)head_dim * 2}) ||
            (has_k && overlap(sqo, Span{k_weight, (uint64_t)head_dim * 2})))
            return fail(QKNR_ERR_ALIAS, "q_out overlaps a weight");
    }
    if (has_k) {
        if (!k_inplace && overlap(sko, sk)) return fail(QKNR_ERR_ALIAS, "k_out overlaps k");
        if (has_q && overlap(sko, sq)) return fail(QKNR_ERR_ALIAS, "k_out overlaps q");
        if (has_q && overlap(sko, sqo)) return fail(QKNR_ERR_ALIAS, "k_out overlaps q_out");
        if (overlap(sko, stab)) return fail(QKNR_ERR_ALIAS, "k_out overlaps rope_table");
        if (overlap(sko, Span{k_weight, (uint64_t)head_dim * 2}) ||
            (has_q && overlap(sko, Span{q_weight, (uint64_t)head_dim * 2})))
            return fail(QKNR_ERR_ALIAS, "k_out overlaps a weight");
    }
    // 2-byte alignment is the minimum for 16-bit element access.
    const uintptr_t any = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                          reinterpret_cast<uintptr_t>(q_out) | reinterpret_cast<uintptr_t>(k_out) |
                          reinterpret_cast<uintptr_t>(q_weight) |
                          reinterpret_cast<uintptr_t>(k_weight);
    if (any & 1u) return fail(QKNR_ERR_ALIGN, "a 16-bit pointer is not 2-byte aligned");
    if (reinterpret_cast<uintptr_t>(rope_table) & (uintptr_t)(tb - 1))
        return fail(QKNR_ERR_ALIGN, "rope_table is not aligned to its element size");

    // ---- device access ----
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    qknr::RopeTableArgs a{};
    const void* p = nullptr;
    int rc;
    if ((rc = classify(rope_table, "rope_table", dev, &p))) return rc;
    a.table = static_cast<const uint8_t*>(p);
    if (has_q) {
        if ((rc = classify(q, "q", dev, &p))) return rc;
        a.q = static_cast<const uint8_t*>(p);
        if ((rc = classify(q_out, "q_out", dev, &p))) return rc;
        a.q_out = static_cast<uint8_t*>(const_cast<void*>(p));
        if ((rc = classify(q_weight, "q_weight", dev, &p))) return rc;
        a.q_weight = static_cast<const uint8_t*>(p);
    }
    if (has_k) {
        if ((rc = classify(k, "k", dev, &p))) return rc;
        a.k = static_cast<const uint8_t*>(p);
        if ((rc = classify(k_out, "k_out", dev, &p))) return rc;
        a.k_out = static_cast<uint8_t*>(const_cast<void*>(p));
        if ((rc = classify(k_weight, "k_weight", dev, &p))) return rc;
        a.k_weight = static_cast<const uint8_t*>(p);
    }
    a.num_tokens = num_tokens;
    a.q_stride = qs;
    a.k_stride = ks;
    a.q_out_stride = qos;
    a.k_out_stride = kos;
    a.hq = heads_q;
    a.hk = heads_k;
    a.head_dim = head_dim;
    a.rotary_dim = R;
    a.table_f32 = table_dtype == QKNR_DT_F32;
    a.act_f16 = act_dtype == QKNR_DT_F16;
    a.interleaved = interleaved ? 1 : 0;
    a.in_place = q_inplace || k_inplace;
    a.eps = eps;
    a.stall_tx_bytes = g_fault_extra_bytes.load(std::memory_order_relaxed);
    a.wait_limit_ns = a.stall_tx_bytes ? g_fault_limit_ns.load() : 0;

    // Fast kernel: 16-byte vectors everywhere and rotation pairs inside a lane.
    const bool vec_ok =
        aligned16(a.table) && (!has_q || (aligned16(a.q) && aligned16(a.q_out) &&
                                          aligned16(a.q_weight) && qs % 8 == 0 && qos % 8 == 0)) &&
        (!has_k || (aligned16(a.k) && aligned16(a.k_out) && aligned16(a.k_weight) &&
                    ks % 8 == 0 && kos % 8 == 0));
    const bool shape_ok = head_dim % 16 == 0 && (interleaved ? R % 8 == 0 : R % 16 == 0);
    qknr::LaunchInfo info{};
    e = qknr::launch_rope_table(a, vec_ok && shape_ok, static_cast<cudaStream_t>(cuda_stream),
                                &info);
    if (e != cudaSuccess) return cuda_fail(e, "table kernel launch");
    return ok();
}

}  // extern "C"

namespace {

// The three 3D entry points share one body. mode: kModeWhole (the full
// transform), kModePartialSsq (per-token sums of squares of this call's Q and
// K heads into ssq_out only), kModeSuppliedSsq (the full transform with the
// per-token sums taken from ssq_in, over heads_q_total / heads_k_total heads).
int run_3d(const qknr_rope_3d_params* prm, int mode, float* ssq_out, const float* ssq_in,
           int32_t heads_q_total, int32_t heads_k_total, void* cuda_stream) {
    if (!prm) return fail(QKNR_ERR_NULL, "params is NULL");
    if (prm->struct_size != sizeof(qknr_rope_3d_params))
        return fail(QKNR_ERR_SHAPE, "params.struct_size %zu != %zu (header mismatch)",
                    prm->struct_size, sizeof(qknr_rope_3d_params));
    const qknr_rope_3d_params& p = *prm;
    const bool partial = mode == qknr::kModePartialSsq;
    const bool supplied = mode == qknr::kModeSuppliedSsq;
    const bool norm = partial || p.is_qk_norm;
    const int D = p.head_dim;
    if (D != 64 && D != 128 && D != 256)
        return fail(QKNR_ERR_SHAPE, "head_dim %d must be 64, 128 or 256", D);
    if (p.num_heads_q < 0 || p.num_heads_k < 0 || p.num_heads_v < 0 ||
        p.num_heads_q + p.num_heads_k + p.num_heads_v < 1)
        return fail(QKNR_ERR_SHAPE, "head counts must be >= 0 with at least one head");
    const int maxh = qknr::rope3d_max_heads(D);
    if (p.num_heads_q > maxh || p.num_heads_k > maxh)
        return fail(QKNR_ERR_UNSUPPORTED, "more than %d Q or K heads of %d channels", maxh, D);
    if (p.ppf < 1 || p.pph < 1 || p.ppw < 1)
        return fail(QKNR_ERR_SHAPE, "ppf, pph and ppw must be >= 1");
    const int64_t P = (int64_t)p.ppf * p.pph * p.ppw;
    if (P > INT32_MAX) return fail(QKNR_ERR_SHAPE, "ppf*pph*ppw exceeds 2^31-1");
    const int cf = p.num_frame_channels, ch = p.num_height_channels, cw = p.num_width_channels;
    if (cf < 0 || ch < 0 || cw < 0 || (cf & 1) || (ch & 1) || (cw & 1))
        return fail(QKNR_ERR_SHAPE, "channel counts must be even and >= 0 (%d/%d/%d)", cf, ch, cw);
    if (cf + ch + cw != D)
        return fail(QKNR_ERR_SHAPE, "channels %d+%d+%d != head_dim %d", cf, ch, cw, D);
    if (p.num_tokens < 0) return fail(QKNR_ERR_SHAPE, "num_tokens < 0");
    if (p.pos_offset < 0) return fail(QKNR_ERR_SHAPE, "pos_offset < 0");
    if (!p.sequence_shard && p.num_tokens % P != 0)
        return fail(QKNR_ERR_SHAPE,
                    "num_tokens %lld not divisible by ppf*pph*ppw = %lld (a slice of a longer "
                    "sequence sets sequence_shard)",
                    (long long)p.num_tokens, (long long)P);
    if (!(p.base > 0.0) || std::isinf(p.base)) return fail(QKNR_ERR_SHAPE, "base must be > 0");
    const bool per_axis = p.neox_per_axis && !p.interleave;
    if (per_axis && ((cf | ch | cw) & 15))
        return fail(QKNR_ERR_UNSUPPORTED,
                    "NeoX pairs per axis group are built for channel groups that are multiples "
                    "of 16 (%d/%d/%d)", cf, ch, cw);
    if (p.factor != 1.0f)
        return fail(QKNR_ERR_UNSUPPORTED, "YARN scaling (factor %g != 1) is not supported",
                    (double)p.factor);
    if (p.attention_factor != 1.0f)
        return fail(QKNR_ERR_SHAPE, "attention_factor other than 1 needs YARN (factor != 1), which is not built");
    if (norm && !partial && (!(p.eps >= 0.0f) || std::isinf(p.eps)))
        return fail(QKNR_ERR_SHAPE, "eps must be >= 0");
    if (!partial && p.output_fp8 &&
        (!std::isfinite(p.output_quant_scale) || !std::isfinite(p.v_quant_scale)))
        return fail(QKNR_ERR_SHAPE, "FP8 scales must be finite");
    if (supplied) {
        if (!p.is_qk_norm) return fail(QKNR_ERR_SHAPE, "supplied sums need is_qk_norm = 1");
        if (heads_q_total < p.num_heads_q || heads_k_total < p.num_heads_k)
            return fail(QKNR_ERR_SHAPE, "heads_*_total (%d, %d) below this slice's heads (%d, %d)",
                        heads_q_total, heads_k_total, p.num_heads_q, p.num_heads_k);
    }
    if (p.num_tokens == 0) return ok();

    const int64_t T = p.num_tokens;
    const int64_t row = (int64_t)(p.num_heads_q + p.num_heads_k + p.num_heads_v) * D;
    const int ob = p.output_fp8 ? 1 : 2;
    const bool hq = p.num_heads_q > 0 && !partial, hk = p.num_heads_k > 0 && !partial;
    const bool hv = p.num_heads_v > 0 && !partial;
    const bool wq = norm && !partial && p.num_heads_q > 0, wk = norm && !partial && p.num_heads_k > 0;
    if (!p.qkv) return fail(QKNR_ERR_NULL, "qkv is NULL");
    if ((hq && !p.q_out) || (hk && !p.k_out) || (hv && !p.v_out))
        return fail(QKNR_ERR_NULL, "an output pointer is NULL");
    if ((wq && !p.q_weight) || (wk && !p.k_weight))
        return fail(QKNR_ERR_NULL, "a weight pointer is NULL with is_qk_norm");
    if (partial && !ssq_out) return fail(QKNR_ERR_NULL, "ssq_out is NULL");
    if (supplied && !ssq_in) return fail(QKNR_ERR_NULL, "ssq is NULL");
    const Span sin_{p.qkv, (uint64_t)T * row * 2};
    const Span so[4] = {{hq ? p.q_out : nullptr, (uint64_t)T * p.num_heads_q * D * ob},
                        {hk ? p.k_out : nullptr, (uint64_t)T * p.num_heads_k * D * ob},
                        {hv ? p.v_out : nullptr, (uint64_t)T * p.num_heads_v * D * ob},
                        {ssq_out, (uint64_t)T * 8}};
    const Span si[3] = {{wq ? p.q_weight : nullptr, (uint64_t)p.num_heads_q * D * 2},
                        {wk ? p.k_weight : nullptr, (uint64_t)p.num_heads_k * D * 2},
                        {ssq_in, (uint64_t)T * 8}};
    for (int i = 0; i < 4; ++i) {
        if (overlap(so[i], sin_)) return fail(QKNR_ERR_ALIAS, "an output overlaps qkv");
        for (int j = 0; j < i; ++j)
            if (overlap(so[i], so[j])) return fail(QKNR_ERR_ALIAS, "two outputs overlap");
        for (int j = 0; j < 3; ++j)
            if (overlap(so[i], si[j])) return fail(QKNR_ERR_ALIAS, "an output overlaps an input");
    }
    if (!aligned16(p.qkv) || (hq && !aligned16(p.q_out)) || (hk && !aligned16(p.k_out)) ||
        (hv && !aligned16(p.v_out)))
        return fail(QKNR_ERR_ALIGN, "qkv and the outputs must be 16-byte aligned");
    if ((wq && !aligned16(p.q_weight)) || (wk && !aligned16(p.k_weight)))
        return fail(QKNR_ERR_ALIGN, "weights must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(ssq_out) | reinterpret_cast<uintptr_t>(ssq_in)) & 7u)
        return fail(QKNR_ERR_ALIGN, "the [T][2] sums must be 8-byte aligned");

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    qknr::Rope3DArgs a{};
    const void* ptr = nullptr;
    int rc;
    if ((rc = classify(p.qkv, "qkv", dev, &ptr))) return rc;
    a.qkv = static_cast<const uint8_t*>(ptr);
    if (hq) {
        if ((rc = classify(p.q_out, "q_out", dev, &ptr))) return rc;
        a.q_out = static_cast<uint8_t*>(const_cast<void*>(ptr));
    }
    if (hk) {
        if ((rc = classify(p.k_out, "k_out", dev, &ptr))) return rc;
        a.k_out = static_cast<uint8_t*>(const_cast<void*>(ptr));
    }
    if (hv) {
        if ((rc = classify(p.v_out, "v_out", dev, &ptr))) return rc;
        a.v_out = static_cast<uint8_t*>(const_cast<void*>(ptr));
    }
    if (wq) {
        if ((rc = classify(p.q_weight, "q_weight", dev, &ptr))) return rc;
        a.q_weight = static_cast<const uint8_t*>(ptr);
    }
    if (wk) {
        if ((rc = classify(p.k_weight, "k_weight", dev, &ptr))) return rc;
        a.k_weight = static_cast<const uint8_t*>(ptr);
    }
    if (partial) {
        if ((rc = classify(ssq_out, "ssq_out", dev, &ptr))) return rc;
        a.ssq_out = static_cast<float*>(const_cast<void*>(ptr));
    }
    if (supplied) {
        if ((rc = classify(ssq_in, "ssq", dev, &ptr))) return rc;
        a.ssq_in = static_cast<const float*>(ptr);
    }
    a.num_tokens = T;
    a.pos_offset = p.pos_offset % P;
    a.ppf = p.ppf;
    a.pph = p.pph;
    a.ppw = p.ppw;
    a.cf = cf;
    a.ch = ch;
    a.cw = cw;
    a.hq = p.num_heads_q;
    a.hk = p.num_heads_k;
    a.hv = p.num_heads_v;
    a.is_qk_norm = norm ? 1 : 0;
    const int64_t entries = (int64_t)p.ppf * (cf / 2) + (int64_t)p.pph * (ch / 2) +
                            (int64_t)p.ppw * (cw / 2);
    a.table_entries = entries > (1 << 20) ? (1 << 20) + 1 : (int32_t)entries;
    a.eps = p.eps;
    a.q_scale = p.output_quant_scale;
    a.v_scale = p.v_quant_scale;
    a.base = p.base;
    a.mode = mode;
    a.neox_per_axis = per_axis ? 1 : 0;
    a.norm_q_elems = (supplied ? heads_q_total : p.num_heads_q) * D;
    a.norm_k_elems = (supplied ? heads_k_total : p.num_heads_k) * D;
    a.stall_tx_bytes = g_fault_extra_bytes.load(std::memory_order_relaxed);
    a.wait_limit_ns = a.stall_tx_bytes ? g_fault_limit_ns.load() : 0;
    qknr::LaunchInfo info{};
    e = qknr::launch_rope3d(a, D, p.interleave ? 0 : 1, (p.output_fp8 && !partial) ? 1 : 0,
                            static_cast<cudaStream_t>(cuda_stream), &info);
    if (e == cudaErrorNotSupported && per_axis) {
        cudaGetLastError();
        return fail(QKNR_ERR_UNSUPPORTED,
                    "the per-axis NeoX layout runs on the register-resident kernel, which does "
                    "not take %d + %d heads of %d (a row of %lld bytes)",
                    p.num_heads_q, p.num_heads_k, D, (long long)(row * 2));
    }
    if (e == cudaErrorNotSupported) {
        cudaGetLastError();
        return fail(QKNR_ERR_UNSUPPORTED,
                    "a row of %lld bytes is too long for the pipelined kernel that the "
                    "tensor-parallel passes need", (long long)(row * 2));
    }
    if (e != cudaSuccess) return cuda_fail(e, "3D kernel launch");
    return ok();
}

}  // namespace

extern "C" {

int qknr_ucpe_cam_prep(const void* q_normed, const void* k_normed, const void* v_raw,
                       const float* proj_q, const float* proj_kv, const float* rope_cos,
                       const float* rope_sin, void* q_trans, void* k_trans, void* v_trans,
                       float* inflation_sq, int32_t act_dtype, int64_t batch,
                       int64_t num_tokens, int32_t num_heads, int32_t head_dim, float k_scale,
                       void* cuda_stream) {
    // ---- shape checks (host only) ----
    if (batch < 0 || num_tokens < 0 || num_heads < 0)
        return fail(QKNR_ERR_SHAPE, "batch, num_tokens and num_heads must be >= 0");
    if (head_dim < 8 || head_dim > 256 || head_dim % 8 != 0)
        return fail(QKNR_ERR_SHAPE, "head_dim %d must be a multiple of 8 from 8 to 256",
                    head_dim);
    if (act_dtype != QKNR_DT_BF16 && act_dtype != QKNR_DT_F16)
        return fail(QKNR_ERR_SHAPE, "activation dtype must be bfloat16 or float16");
    if (!std::isfinite(k_scale)) return fail(QKNR_ERR_SHAPE, "k_scale must be finite");
    // Element counts must fit int64 comfortably (the kernel indexes in int64).
    const int64_t kLimit = (int64_t)1 << 50;
    if (batch > 0 && num_tokens > 0 && num_heads > 0 &&
        (double)batch * (double)num_tokens * (double)num_heads * (double)head_dim > (double)kLimit)
        return fail(QKNR_ERR_SHAPE, "tensor too large");
    if (batch == 0 || num_tokens == 0 || num_heads == 0) return ok();

    // ---- pointers ----
    if (!q_normed || !k_normed || !v_raw) return fail(QKNR_ERR_NULL, "q_normed, k_normed or v_raw is NULL");
    if (!proj_q || !proj_kv) return fail(QKNR_ERR_NULL, "proj_q or proj_kv is NULL");
    if (!rope_cos || !rope_sin) return fail(QKNR_ERR_NULL, "rope_cos or rope_sin is NULL");
    if (!q_trans || !k_trans || !v_trans) return fail(QKNR_ERR_NULL, "q_trans, k_trans or v_trans is NULL");
    const void* all[] = {q_normed, k_normed, v_raw, proj_q, proj_kv, rope_cos, rope_sin,
                         q_trans, k_trans, v_trans, inflation_sq};
    for (const void* ptr : all)
        if (ptr && !aligned16(ptr)) return fail(QKNR_ERR_ALIGN, "a pointer is not 16-byte aligned");
    const uint64_t act_bytes = (uint64_t)batch * num_tokens * num_heads * head_dim * 2;
    const uint64_t proj_bytes = (uint64_t)batch * num_tokens * 64;
    const uint64_t rope_bytes = (uint64_t)num_tokens * (head_dim / 2) * 4;
    const Span ins[] = {{q_normed, act_bytes}, {k_normed, act_bytes}, {v_raw, act_bytes},
                        {proj_q, proj_bytes},  {proj_kv, proj_bytes}, {rope_cos, rope_bytes},
                        {rope_sin, rope_bytes}};
    const Span outs[] = {{q_trans, act_bytes},
                         {k_trans, act_bytes},
                         {v_trans, act_bytes},
                         {inflation_sq, (uint64_t)batch * num_heads * num_tokens * 4}};
    for (int i = 0; i < 4; ++i) {
        for (const Span& in : ins)
            if (overlap(outs[i], in)) return fail(QKNR_ERR_ALIAS, "an output overlaps an input");
        for (int j = 0; j < i; ++j)
            if (overlap(outs[i], outs[j])) return fail(QKNR_ERR_ALIAS, "two outputs overlap");
    }

    // ---- device access ----
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    const char* names[] = {"q_normed", "k_normed", "v_raw", "proj_q", "proj_kv", "rope_cos",
                           "rope_sin", "q_trans", "k_trans", "v_trans", "inflation_sq"};
    const void* dp[11] = {};
    for (int i = 0; i < 11; ++i) {
        if (!all[i]) continue;
        int rc = classify(all[i], names[i], dev, &dp[i]);
        if (rc) return rc;
        if (!aligned16(dp[i])) return fail(QKNR_ERR_ALIGN, "%s: device address not 16-byte aligned", names[i]);
    }
    qknr::UcpeArgs a{};
    a.q = static_cast<const uint8_t*>(dp[0]);
    a.k = static_cast<const uint8_t*>(dp[1]);
    a.v = static_cast<const uint8_t*>(dp[2]);
    a.proj_q = static_cast<const float*>(dp[3]);
    a.proj_kv = static_cast<const float*>(dp[4]);
    a.rope_cos = static_cast<const float*>(dp[5]);
    a.rope_sin = static_cast<const float*>(dp[6]);
    a.q_out = static_cast<uint8_t*>(const_cast<void*>(dp[7]));
    a.k_out = static_cast<uint8_t*>(const_cast<void*>(dp[8]));
    a.v_out = static_cast<uint8_t*>(const_cast<void*>(dp[9]));
    a.inflation_sq = static_cast<float*>(const_cast<void*>(dp[10]));
    a.batch = batch;
    a.num_tokens = num_tokens;
    a.heads = num_heads;
    a.head_dim = head_dim;
    a.act_f16 = act_dtype == QKNR_DT_F16;
    a.k_scale = k_scale;
    qknr::UcpeControl ctl{};
    ctl.stall_tx_bytes = g_fault_extra_bytes.load(std::memory_order_relaxed);
    ctl.wait_limit_ns = ctl.stall_tx_bytes ? g_fault_limit_ns.load() : 2000000000ull;  // 2 s
    // The warp-specialised kernel reads q, k and v through tensor maps: only
    // for device memory (page-locked host or managed buffers take another).
    ctl.device_inputs = 1;
    for (int i = 0; i < 3; ++i) {
        cudaPointerAttributes attr;
        if (cudaPointerGetAttributes(&attr, all[i]) != cudaSuccess) {
            cudaGetLastError();
            ctl.device_inputs = 0;
        } else if (attr.type != cudaMemoryTypeDevice) {
            ctl.device_inputs = 0;
        }
    }
    qknr::LaunchInfo info{};
    e = qknr::launch_ucpe(a, ctl, static_cast<cudaStream_t>(cuda_stream), &info);
    if (e != cudaSuccess) return cuda_fail(e, "camera prep kernel launch");
    return ok();
}

int qknr_rope_3d(const qknr_rope_3d_params* prm, void* cuda_stream) {
    return run_3d(prm, qknr::kModeWhole, nullptr, nullptr, 0, 0, cuda_stream);
}

int qknr_rope_3d_partial_ssq(const qknr_rope_3d_params* prm, float* ssq_out, void* cuda_stream) {
    return run_3d(prm, qknr::kModePartialSsq, ssq_out, nullptr, 0, 0, cuda_stream);
}

int qknr_rope_3d_with_ssq(const qknr_rope_3d_params* prm, const float* ssq,
                          int32_t heads_q_total, int32_t heads_k_total, void* cuda_stream) {
    return run_3d(prm, qknr::kModeSuppliedSsq, nullptr, ssq, heads_q_total, heads_k_total,
                  cuda_stream);
}

}  // extern "C"
