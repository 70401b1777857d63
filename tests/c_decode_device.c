/* Plain C11 use of include/pagedattn.h on a GPU: reads one decode problem from
 * binary files, puts it in device memory with the CUDA runtime, calls
 * pa_workspace_size and pa_decode, and writes dst back to a file.
 * tests/test_gpu_c_program.py builds it with gcc, writes the inputs, and
 * compares its dst with the same call made through the Python binding.
 *
 *   c_decode_device <dir>
 *
 * <dir>/dims.txt holds: batch H_q H_kv head_dim block_size num_blocks
 * max_blocks_per_seq window scale(float) max_span max_query_len num_tokens;
 * q.bin (bf16), k.bin, v.bin (bf16 caches), tables.bin, seq_lens.bin,
 * query_lens.bin (int32) hold the arrays; dst.bin is written. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "pagedattn.h"

static void *read_file(const char *dir, const char *name, size_t *bytes)
{
    char path[1024];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "rb");
    if (!f) return NULL;
    fseek(f, 0, SEEK_END);
    const long n = ftell(f);
    fseek(f, 0, SEEK_SET);
    void *buf = malloc(n > 0 ? (size_t)n : 1u);
    if (buf && n > 0 && fread(buf, 1, (size_t)n, f) != (size_t)n) {
        free(buf);
        buf = NULL;
    }
    fclose(f);
    *bytes = (size_t)n;
    return buf;
}

static void *to_device(const void *host, size_t bytes)
{
    void *d = NULL;
    if (cudaMalloc(&d, bytes ? bytes : 16u) != cudaSuccess) return NULL;
    if (bytes && cudaMemcpy(d, host, bytes, cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
    return d;
}

int main(int argc, char **argv)
{
    if (argc != 2) {
        fprintf(stderr, "usage: %s <dir>\n", argv[0]);
        return 2;
    }
    const char *dir = argv[1];
    char path[1024];
    snprintf(path, sizeof path, "%s/dims.txt", dir);
    FILE *f = fopen(path, "r");
    if (!f) return 3;
    int batch, hq, hkv, d, bs, nblocks, mbps, window, span, qlen, ntok;
    float scale;
    if (fscanf(f, "%d %d %d %d %d %d %d %d %f %d %d %d", &batch, &hq, &hkv, &d, &bs, &nblocks,
               &mbps, &window, &scale, &span, &qlen, &ntok) != 12) {
        fclose(f);
        return 4;
    }
    fclose(f);

    const char *names[6] = {"q.bin", "k.bin", "v.bin", "tables.bin", "seq_lens.bin",
                            "query_lens.bin"};
    void *host[6], *dev[6];
    size_t bytes[6];
    for (int i = 0; i < 6; ++i) {
        host[i] = read_file(dir, names[i], &bytes[i]);
        if (!host[i]) return 5;
        dev[i] = to_device(host[i], bytes[i]);
        if (!dev[i]) return 6;
    }

    pa_params p;
    memset(&p, 0, sizeof p);
    p.batch = batch;
    p.num_q_heads = hq;
    p.num_kv_heads = hkv;
    p.head_dim = d;
    p.num_blocks = nblocks;
    p.max_blocks_per_seq = mbps;
    p.max_span_hint = span;
    p.max_query_len_hint = qlen;
    const size_t ws_bytes = pa_workspace_size(&p, bs);
    if (ws_bytes == (size_t)-1) {
        fprintf(stderr, "workspace size: %s\n", pa_last_error());
        return 7;
    }
    void *ws = NULL;
    if (ws_bytes && cudaMalloc(&ws, ws_bytes) != cudaSuccess) return 8;
    p.workspace = ws;
    p.workspace_bytes = ws_bytes;

    const size_t dst_bytes = (size_t)ntok * hq * d * 2;
    void *dst = NULL;
    if (cudaMalloc(&dst, dst_bytes) != cudaSuccess) return 9;
    cudaStream_t stream;
    if (cudaStreamCreate(&stream) != cudaSuccess) return 10;
    const int rc = pa_decode(dst, dev[0], dev[1], dev[2], (const int32_t *)dev[3],
                             (const int32_t *)dev[4], (const int32_t *)dev[5], scale, window, bs,
                             &p, stream);
    if (rc != PA_OK) {
        fprintf(stderr, "pa_decode: %d %s\n", rc, pa_last_error());
        return 11;
    }
    unsigned int status = 1;
    if (pa_device_status(&status, 1, stream) != PA_OK || status != 0) return 12;
    void *out = malloc(dst_bytes);
    if (!out || cudaMemcpy(out, dst, dst_bytes, cudaMemcpyDeviceToHost) != cudaSuccess) return 13;
    snprintf(path, sizeof path, "%s/dst.bin", dir);
    FILE *o = fopen(path, "wb");
    if (!o || fwrite(out, 1, dst_bytes, o) != dst_bytes) return 14;
    fclose(o);
    printf("ok %zu workspace bytes\n", ws_bytes);
    for (int i = 0; i < 6; ++i) {
        cudaFree(dev[i]);
        free(host[i]);
    }
    cudaFree(ws);
    cudaFree(dst);
    free(out);
    cudaStreamDestroy(stream);
    return 0;
}
