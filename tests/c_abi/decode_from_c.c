/*
 * decode_from_c.c -- a C consumer of liblca_b200.so, with no Python in the
 * way: plain device pointers from cudaMalloc, the caller-owned workspace
 * sized by lca_workspace_bytes, one lca_decode step on the legacy default
 * stream, the library's status codes and its device status word.
 *
 * Usage: decode_from_c B L dir
 *   reads  dir/cache.bin    [B][L][576] bf16
 *          dir/q_recent.bin [B][16][16][576] bf16
 *          dir/q.bin        [B][16][576] bf16
 *          dir/w_uv.bin     [16][512][128] bf16
 *   writes dir/out.bin      [B][16][128] fp32
 * Exit status 0 on success; a message on stderr otherwise.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "lca.h"

static void *read_file(const char *dir, const char *name, size_t bytes)
{
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "rb");
    if (!f) return NULL;
    void *buf = malloc(bytes);
    size_t got = buf ? fread(buf, 1, bytes, f) : 0;
    fclose(f);
    if (got != bytes) {
        free(buf);
        return NULL;
    }
    return buf;
}

static void *to_device(const void *host, size_t bytes)
{
    void *d = NULL;
    if (cudaMalloc(&d, bytes) != cudaSuccess) return NULL;
    if (cudaMemcpy(d, host, bytes, cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
    return d;
}

#define FAIL(...)                         \
    do {                                  \
        fprintf(stderr, __VA_ARGS__);     \
        fputc('\n', stderr);              \
        return 1;                         \
    } while (0)

int main(int argc, char **argv)
{
    if (argc != 4) FAIL("usage: %s B L dir", argv[0]);
    const int B = atoi(argv[1]);
    const int64_t L = atoll(argv[2]);
    const char *dir = argv[3];
    const size_t n_cache = (size_t)B * (size_t)L * LCA_D * 2, n_qr = (size_t)B * 16 * LCA_HEADS * LCA_D * 2;
    const size_t n_q = (size_t)B * LCA_HEADS * LCA_D * 2, n_w = (size_t)LCA_HEADS * LCA_DC * LCA_DV * 2;
    const size_t n_out = (size_t)B * LCA_HEADS * LCA_DV * 4;

    void *h_cache = read_file(dir, "cache.bin", n_cache), *h_qr = read_file(dir, "q_recent.bin", n_qr);
    void *h_q = read_file(dir, "q.bin", n_q), *h_w = read_file(dir, "w_uv.bin", n_w);
    if (!h_cache || !h_qr || !h_q || !h_w) FAIL("cannot read the inputs in %s", dir);
    void *d_cache = to_device(h_cache, n_cache), *d_qr = to_device(h_qr, n_qr);
    void *d_q = to_device(h_q, n_q), *d_w = to_device(h_w, n_w);
    float *d_out = NULL;
    if (!d_cache || !d_qr || !d_q || !d_w || cudaMalloc((void **)&d_out, n_out) != cudaSuccess)
        FAIL("device allocation failed");

    lca_params p;
    memset(&p, 0, sizeof p);
    p.g = 16;
    p.w = 1024;
    p.scale = (float)(1.0 / sqrt(192.0));
    p.variant = LCA_VARIANT_LCA;
    p.cache_pitch = 0;   /* packed [B][L][576] */

    const size_t ws_bytes = lca_workspace_bytes(LCA_OP_DECODE, B, L, 0, p);
    void *d_ws = NULL;
    if (ws_bytes == 0 || cudaMalloc(&d_ws, ws_bytes) != cudaSuccess) FAIL("workspace of %zu bytes", ws_bytes);

    /* an invalid argument is rejected before anything is launched */
    lca_params bad = p;
    bad.scale = -1.0f;
    int rc = lca_decode(d_cache, d_qr, d_q, d_w, B, L, bad, d_out, NULL, NULL, d_ws, ws_bytes, NULL);
    if (rc != LCA_ERR_INVALID_ARG) FAIL("bad scale gave %d (%s)", rc, lca_strerror(rc));
    rc = lca_decode(d_cache, d_qr, d_q, d_w, B, L, p, d_out, NULL, NULL, d_ws, ws_bytes / 2, NULL);
    if (rc != LCA_ERR_WORKSPACE) FAIL("small workspace gave %d (%s)", rc, lca_strerror(rc));

    rc = lca_decode(d_cache, d_qr, d_q, d_w, B, L, p, d_out, NULL, NULL, d_ws, ws_bytes, NULL);
    if (rc != LCA_OK) FAIL("lca_decode: %s", lca_strerror(rc));
    int detail = 0;
    rc = lca_device_status(1, &detail);   /* synchronises the device */
    if (rc != LCA_OK) FAIL("device status %d, detail %#x", rc, detail);

    float *h_out = (float *)malloc(n_out);
    if (!h_out || cudaMemcpy(h_out, d_out, n_out, cudaMemcpyDeviceToHost) != cudaSuccess) FAIL("copy back");
    char path[4096];
    snprintf(path, sizeof path, "%s/out.bin", dir);
    FILE *f = fopen(path, "wb");
    if (!f || fwrite(h_out, 1, n_out, f) != n_out) FAIL("cannot write %s", path);
    fclose(f);
    printf("lca_decode from C: B=%d L=%lld, %zu workspace bytes, %lld kernel launches\n", B, (long long)L,
           ws_bytes, (long long)lca_launch_count());
    cudaFree(d_cache), cudaFree(d_qr), cudaFree(d_q), cudaFree(d_w), cudaFree(d_out), cudaFree(d_ws);
    free(h_cache), free(h_qr), free(h_q), free(h_w), free(h_out);
    return 0;
}
