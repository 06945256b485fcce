/* A plain C program that runs one MoE layer forward on the GPU through the library's C ABI
 * (include/moe.h), with device memory from cudaMalloc: no Python, no torch.
 *
 *   moe_c_gpu <dir> T D E F k
 *
 * Reads the layer's inputs from <dir> as raw little-endian bf16 arrays (x.bin [T,D],
 * wg.bin [E,D], wgate.bin and wup.bin [E,F,D], wdown.bin [E,D,F]), describes a softmax top-k
 * renormalised, dropless, SwiGLU layer ("Top-k 路由" gate Steps 1-3; Tiny MoE sections 3-6),
 * sizes and allocates the workspace, calls moe_layer_forward on a stream of its own, reads the
 * device error word, and writes the layer output to <dir>/out.bin (bf16 [T,D]) and the balance
 * statistics (moe_stats_t) to <dir>/stats.bin.  Exit status 0 on success; any failed CUDA or
 * library call prints its error and exits 1. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "moe.h"

static void die_cuda(cudaError_t e, const char* what) {
    if (e != cudaSuccess) {
        fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
        exit(1);
    }
}

static void die_moe(moe_status_t s, const char* what) {
    if (s != MOE_OK) {
        fprintf(stderr, "%s: %s\n", what, moe_status_string(s));
        exit(1);
    }
}

static void* read_to_device(const char* dir, const char* name, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "rb");
    if (!f) {
        fprintf(stderr, "cannot open %s\n", path);
        exit(1);
    }
    void* host = malloc(bytes);
    if (!host || fread(host, 1, bytes, f) != bytes) {
        fprintf(stderr, "short read of %s\n", path);
        exit(1);
    }
    fclose(f);
    void* dev = NULL;
    die_cuda(cudaMalloc(&dev, bytes), "cudaMalloc");
    die_cuda(cudaMemcpy(dev, host, bytes, cudaMemcpyHostToDevice), "cudaMemcpy H2D");
    free(host);
    return dev;
}

static void write_from_device(const char* dir, const char* name, const void* dev, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    void* host = malloc(bytes);
    if (!host) exit(1);
    die_cuda(cudaMemcpy(host, dev, bytes, cudaMemcpyDeviceToHost), "cudaMemcpy D2H");
    FILE* f = fopen(path, "wb");
    if (!f || fwrite(host, 1, bytes, f) != bytes) {
        fprintf(stderr, "cannot write %s\n", path);
        exit(1);
    }
    fclose(f);
    free(host);
}

int main(int argc, char** argv) {
    if (argc != 7) {
        fprintf(stderr, "usage: %s <dir> T D E F k\n", argv[0]);
        return 2;
    }
    const char* dir = argv[1];
    moe_desc_t d;
    memset(&d, 0, sizeof d);
    d.T = atoi(argv[2]); d.D = atoi(argv[3]); d.E = atoi(argv[4]); d.F = atoi(argv[5]);
    d.k = atoi(argv[6]);
    d.score = MOE_SCORE_SOFTMAX; d.select = MOE_TOKEN_CHOICE; d.gate = MOE_GATE_RENORM;
    d.overflow = MOE_DROPLESS; d.act = MOE_ACT_SWIGLU; d.dtype = MOE_BF16;
    d.aux_alpha = 0.01f; d.n_group = 1; d.topk_group = 1;

    const size_t es = 2;   /* bf16 */
    const size_t T = (size_t)d.T, D = (size_t)d.D, E = (size_t)d.E, F = (size_t)d.F;
    void* x = read_to_device(dir, "x.bin", T * D * es);
    void* wg = read_to_device(dir, "wg.bin", E * D * es);
    void* wgate = read_to_device(dir, "wgate.bin", E * F * D * es);
    void* wup = read_to_device(dir, "wup.bin", E * F * D * es);
    void* wdown = read_to_device(dir, "wdown.bin", E * D * F * es);
    void* out = NULL;
    die_cuda(cudaMalloc(&out, T * D * es), "cudaMalloc out");

    size_t ws_bytes = 0;
    die_moe(moe_workspace_size(&d, &ws_bytes), "moe_workspace_size");
    void* ws = NULL;
    die_cuda(cudaMalloc(&ws, ws_bytes), "cudaMalloc workspace");
    cudaStream_t stream;
    die_cuda(cudaStreamCreate(&stream), "cudaStreamCreate");

    die_moe(moe_layer_forward(&d, x, wg, NULL, wgate, wup, wdown, NULL, NULL, NULL, out, ws,
                              ws_bytes, (moe_stream_t)stream),
            "moe_layer_forward");
    int32_t code = 0;
    die_moe(moe_get_device_error((moe_stream_t)stream, &code), "moe_get_device_error");
    if (code != 0) {
        fprintf(stderr, "device error word %#x\n", (unsigned)code);
        return 1;
    }

    /* the statistics the layer left in its workspace */
    moe_layer_views_t v;
    die_moe(moe_layer_views(&d, ws, ws_bytes, &v), "moe_layer_views");
    write_from_device(dir, "out.bin", out, T * D * es);
    write_from_device(dir, "stats.bin", v.stats, sizeof(moe_stats_t));
    printf("moe_layer_forward T=%d D=%d E=%d F=%d k=%d: ok (workspace %zu B)\n", d.T, d.D, d.E,
           d.F, d.k, ws_bytes);

    cudaStreamDestroy(stream);
    cudaFree(ws); cudaFree(out); cudaFree(wdown); cudaFree(wup); cudaFree(wgate);
    cudaFree(wg); cudaFree(x);
    return 0;
}
