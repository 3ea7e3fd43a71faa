/*
 * Host cost per call of libqknr.so's two contract entry points, measured from
 * C through the ABI (no Python in the way).
 *
 *   host_cost <3d|table> <tokens> <calls>
 *
 * Shapes per token: "3d" is the FP8 NeoX video geometry of the 3D form
 * (24 + 24 + 24 heads of 128, grid 31 x 24 x 40, channels 32/48/48, E4M3 out;
 * a sequence shard from patch 0, so any token count); "table" is the
 * half-split table form (32 + 8 heads of 128, rotary_dim 96, fp32 table).
 * Buffers are device memory filled with small values; their contents do not
 * change the work a call does.
 *
 * Prints one JSON line:
 *   host_us_per_call    host time of one call: `calls` calls queued back to
 *                       back without synchronising (validation, pointer
 *                       checks and the launch), over `calls`;
 *   device_us_per_call  GPU time of one call with no host in the way: the
 *                       same calls captured once in a CUDA graph and replayed,
 *                       timed with events;
 *   wall_us_per_call    one call and a stream synchronisation, end to end.
 * When device_us_per_call is below host_us_per_call, calls issued back to back
 * keep the GPU waiting on the host: the call is host-bound at that size.
 */
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <time.h>

#include "qknr.h"

static double now_us(void) {
    struct timespec ts;
    clock_gettime(CLOCK_MONOTONIC, &ts);
    return ts.tv_sec * 1e6 + ts.tv_nsec * 1e-3;
}

#define CK(x)                                                                    \
    do {                                                                         \
        cudaError_t e_ = (x);                                                    \
        if (e_ != cudaSuccess) {                                                 \
            fprintf(stderr, "%s:%d %s: %s\n", __FILE__, __LINE__, #x,            \
                    cudaGetErrorString(e_));                                     \
            exit(2);                                                             \
        }                                                                        \
    } while (0)

static void* dev_fill(size_t bytes) {
    void* p = NULL;
    CK(cudaMalloc(&p, bytes ? bytes : 16));
    CK(cudaMemset(p, 0x3c, bytes ? bytes : 16)); /* bf16 0x3c3c ~ 0.011, e4m3 0x3c = 1.5 */
    return p;
}

typedef struct {
    int form_3d;
    qknr_rope_3d_params p3;
    const void *q, *k, *qw, *kw, *tab;
    void *qo, *ko;
    int64_t T;
    cudaStream_t st;
} Call;

static int call_once(Call* c) {
    if (c->form_3d) return qknr_rope_3d(&c->p3, c->st);
    return qknr_rope_table(c->q, c->k, c->qo, c->ko, c->qw, c->kw, c->tab, QKNR_DT_F32,
                           QKNR_DT_BF16, c->T, 32, 8, 128, 96, 0, 0, 0, 0, 1e-6f, 0, c->st);
}

int main(int argc, char** argv) {
    if (argc != 4) {
        fprintf(stderr, "usage: %s <3d|table> <tokens> <calls>\n", argv[0]);
        return 1;
    }
    Call c;
    memset(&c, 0, sizeof(c));
    c.form_3d = strcmp(argv[1], "3d") == 0;
    c.T = atoll(argv[2]);
    const int calls = atoi(argv[3]);
    if (c.T < 1 || calls < 1 || (!c.form_3d && strcmp(argv[1], "table") != 0)) return 1;
    CK(cudaStreamCreateWithFlags(&c.st, cudaStreamNonBlocking));
    const int D = 128;
    if (c.form_3d) {
        const int H = 24;
        qknr_rope_3d_params* p = &c.p3;
        p->struct_size = sizeof(*p);
        p->qkv = dev_fill((size_t)c.T * 3 * H * D * 2);
        p->q_weight = dev_fill((size_t)H * D * 2);
        p->k_weight = dev_fill((size_t)H * D * 2);
        p->q_out = dev_fill((size_t)c.T * H * D);
        p->k_out = dev_fill((size_t)c.T * H * D);
        p->v_out = dev_fill((size_t)c.T * H * D);
        p->num_tokens = c.T;
        p->pos_offset = 0;
        p->ppf = 31; p->pph = 24; p->ppw = 40;
        p->num_frame_channels = 32; p->num_height_channels = 48; p->num_width_channels = 48;
        p->num_heads_q = p->num_heads_k = p->num_heads_v = H;
        p->head_dim = D;
        p->eps = 1e-6f;
        p->base = 10000.0;
        p->interleave = 0;
        p->factor = 1.0f; p->attention_factor = 1.0f;
        p->is_qk_norm = 1;
        p->output_fp8 = 1;
        p->output_quant_scale = 0.5f;
        p->v_quant_scale = 0.25f;
        p->sequence_shard = 1;
    } else {
        c.q = dev_fill((size_t)c.T * 32 * D * 2);
        c.k = dev_fill((size_t)c.T * 8 * D * 2);
        c.qo = dev_fill((size_t)c.T * 32 * D * 2);
        c.ko = dev_fill((size_t)c.T * 8 * D * 2);
        c.qw = dev_fill(D * 2);
        c.kw = dev_fill(D * 2);
        c.tab = dev_fill((size_t)c.T * 96 * 4);
    }
    CK(cudaDeviceSynchronize());
    for (int i = 0; i < 50; ++i) {
        const int rc = call_once(&c);
        if (rc) {
            fprintf(stderr, "call failed: %s (%s)\n", qknr_status_string(rc),
                    qknr_last_error_detail());
            return 3;
        }
    }
    CK(cudaStreamSynchronize(c.st));

    /* host cost: queue `calls` calls, then wait */
    double t0 = now_us();
    for (int i = 0; i < calls; ++i) call_once(&c);
    const double host_us = (now_us() - t0) / calls;
    CK(cudaStreamSynchronize(c.st));

    /* device time: the same calls from a graph */
    cudaGraph_t g;
    cudaGraphExec_t ge;
    CK(cudaStreamBeginCapture(c.st, cudaStreamCaptureModeThreadLocal));
    for (int i = 0; i < calls; ++i) call_once(&c);
    CK(cudaStreamEndCapture(c.st, &g));
    CK(cudaGraphInstantiate(&ge, g, 0));
    CK(cudaGraphLaunch(ge, c.st));
    CK(cudaStreamSynchronize(c.st));
    cudaEvent_t e0, e1;
    CK(cudaEventCreate(&e0));
    CK(cudaEventCreate(&e1));
    CK(cudaEventRecord(e0, c.st));
    CK(cudaGraphLaunch(ge, c.st));
    CK(cudaEventRecord(e1, c.st));
    CK(cudaEventSynchronize(e1));
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, e0, e1));
    const double device_us = ms * 1e3 / calls;

    /* one call end to end */
    const int reps = calls < 200 ? calls : 200;
    t0 = now_us();
    for (int i = 0; i < reps; ++i) {
        call_once(&c);
        cudaStreamSynchronize(c.st);
    }
    const double wall_us = (now_us() - t0) / reps;

    printf("{\"form\": \"%s\", \"tokens\": %lld, \"calls\": %d, \"host_us_per_call\": %.3f, "
           "\"device_us_per_call\": %.3f, \"wall_us_per_call\": %.3f}\n",
           c.form_3d ? "3d" : "table", (long long)c.T, calls, host_us, device_us, wall_us);
    CK(cudaGraphExecDestroy(ge));
    CK(cudaGraphDestroy(g));
    return 0;
}
