/*
 * A plain C client of libsinkrouter.so, compiled against include/sinkrouter.h
 * only (no Python, no C++). Used by tests/test_c_abi.py.
 *
 *   sr_abi_client host
 *       Host-side checks that need no GPU: status strings, workspace sizing
 *       and argument validation (these calls launch nothing).
 *   sr_abi_client gpu <in.bin> <out.bin>
 *       One routed decode step through sr_route and sr_decode_attention on
 *       device buffers this program allocates with the CUDA runtime. in.bin:
 *       int32 header {B, Hq, Hkv, Lmax, tau_bits}, then q, k_cache, v_cache,
 *       k0, v0 (bf16 bit patterns, layouts as in sinkrouter.h) and seq_lens
 *       (int32 [B]). out.bin: out (bf16 [B, Hq, 128]), route_mask (uint8
 *       [B*Hkv]), active_list (int32 [1 + B*Hkv]), device error word (int32).
 * Exit status 0 on success; a message on stderr otherwise.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "sinkrouter.h"
#include <cuda_runtime_api.h> /* the CUDA runtime's C API (device buffers of this client) */

static int fail(const char *what)
{
    fprintf(stderr, "sr_abi_client: %s\n", what);
    return 1;
}

#define CHECK(cond, what)                                                                                  \
    do {                                                                                                   \
        if (!(cond))                                                                                       \
            return fail(what);                                                                             \
    } while (0)

static int host_checks(void)
{
    sr_dims d = {1, 32, 8, 128, 4096};
    CHECK(strcmp(sr_status_string(SR_OK), "SR_OK") == 0, "status string of SR_OK");
    CHECK(sr_decode_workspace_bytes(&d, 0) > 0, "workspace bytes for valid dims");
    CHECK(sr_decode_workspace_bytes(&d, 64) >= sr_decode_workspace_bytes(&d, 0), "forced splits need no less");
    CHECK(sr_decode_workspace_bytes(NULL, 0) == 0, "workspace bytes for NULL dims");
    sr_dims bad = d;
    bad.head_dim = 64;
    CHECK(sr_decode_workspace_bytes(&bad, 0) == 0, "workspace bytes for head_dim 64");
    void *fake = (void *)(uintptr_t)0x10000; /* aligned, never dereferenced */
    CHECK(sr_route(NULL, fake, fake, 0.6f, fake, fake, NULL) == SR_ERR_INVALID_ARG, "sr_route NULL dims");
    CHECK(sr_route(&bad, fake, fake, 0.6f, fake, fake, NULL) == SR_ERR_UNSUPPORTED, "sr_route head_dim 64");
    CHECK(sr_route(&d, NULL, fake, 0.6f, fake, fake, NULL) == SR_ERR_INVALID_ARG, "sr_route NULL q");
    CHECK(sr_decode_attention(&d, fake, fake, fake, fake, fake, fake, fake, 0, fake, NULL, 1u << 30, NULL) ==
              SR_ERR_WORKSPACE,
          "sr_decode_attention NULL workspace");
    CHECK(sr_decode_attention(&d, fake, fake, fake, fake, fake, fake, fake, -1, fake, fake, 1u << 30, NULL) ==
              SR_ERR_INVALID_ARG,
          "sr_decode_attention negative n_splits");
    CHECK(sr_combine_partials(&d, 0, fake, fake, 4128, fake, NULL) == SR_ERR_INVALID_ARG, "combine with 0 parts");
    printf("host checks ok\n");
    return 0;
}

static void *read_all(FILE *f, size_t n)
{
    void *p = malloc(n ? n : 1);
    if (p && n && fread(p, 1, n, f) != n) {
        free(p);
        return NULL;
    }
    return p;
}

static int gpu_step(const char *in_path, const char *out_path)
{
    FILE *f = fopen(in_path, "rb");
    CHECK(f, "cannot open input");
    int32_t hdr[5];
    CHECK(fread(hdr, sizeof hdr, 1, f) == 1, "short header");
    const int B = hdr[0], Hq = hdr[1], Hkv = hdr[2], L = hdr[3];
    float tau;
    memcpy(&tau, &hdr[4], sizeof tau);
    const size_t nq = (size_t)B * Hq * 128 * 2, nkv = (size_t)B * Hkv * L * 128 * 2, n0 = (size_t)B * Hkv * 128 * 2;
    const size_t ns = (size_t)B * 4, U = (size_t)B * Hkv;
    void *h_q = read_all(f, nq), *h_k = read_all(f, nkv), *h_v = read_all(f, nkv);
    void *h_k0 = read_all(f, n0), *h_v0 = read_all(f, n0), *h_sl = read_all(f, ns);
    fclose(f);
    CHECK(h_q && h_k && h_v && h_k0 && h_v0 && h_sl, "short input");

    sr_dims d = {B, Hq, Hkv, 128, L};
    const size_t wsb = sr_decode_workspace_bytes(&d, 0);
    CHECK(wsb > 0, "unsupported dims");
    void *q, *k, *v, *k0, *v0, *sl, *mask, *act, *out, *ws;
    void **dev[] = {&q, &k, &v, &k0, &v0, &sl, &mask, &act, &out, &ws};
    const size_t bytes[] = {nq, nkv, nkv, n0, n0, ns, U, 4 * (U + 1), nq, wsb};
    for (int i = 0; i < 10; ++i)
        CHECK(cudaMalloc(dev[i], bytes[i]) == cudaSuccess, "cudaMalloc");
    const void *host_in[] = {h_q, h_k, h_v, h_k0, h_v0, h_sl};
    for (int i = 0; i < 6; ++i)
        CHECK(cudaMemcpy(*dev[i], host_in[i], bytes[i], cudaMemcpyHostToDevice) == cudaSuccess, "copy in");
    sr_status st = sr_workspace_init(ws, wsb, NULL);
    CHECK(st == SR_OK, sr_status_string(st));
    st = sr_route(&d, q, k0, tau, (uint8_t *)mask, (int32_t *)act, NULL);
    CHECK(st == SR_OK, sr_status_string(st));
    st = sr_decode_attention(&d, q, k, v, k0, v0, (const int32_t *)sl, (const int32_t *)act, 0, out, ws, wsb, NULL);
    CHECK(st == SR_OK, sr_status_string(st));
    CHECK(cudaDeviceSynchronize() == cudaSuccess, "kernel failure");
    int32_t derr = -1;
    st = sr_get_device_error(ws, &derr, NULL);
    CHECK(st == SR_OK, sr_status_string(st));

    void *h_out = malloc(nq), *h_mask = malloc(U), *h_act = malloc(4 * (U + 1));
    CHECK(h_out && h_mask && h_act, "malloc");
    CHECK(cudaMemcpy(h_out, out, nq, cudaMemcpyDeviceToHost) == cudaSuccess, "copy out");
    CHECK(cudaMemcpy(h_mask, mask, U, cudaMemcpyDeviceToHost) == cudaSuccess, "copy out");
    CHECK(cudaMemcpy(h_act, act, 4 * (U + 1), cudaMemcpyDeviceToHost) == cudaSuccess, "copy out");
    FILE *g = fopen(out_path, "wb");
    CHECK(g, "cannot open output");
    CHECK(fwrite(h_out, 1, nq, g) == nq && fwrite(h_mask, 1, U, g) == U && fwrite(h_act, 4, U + 1, g) == U + 1 &&
              fwrite(&derr, 4, 1, g) == 1,
          "write output");
    fclose(g);
    for (int i = 0; i < 10; ++i)
        cudaFree(*dev[i]);
    free(h_q), free(h_k), free(h_v), free(h_k0), free(h_v0), free(h_sl), free(h_out), free(h_mask), free(h_act);
    printf("gpu step ok\n");
    return 0;
}

int main(int argc, char **argv)
{
    if (argc >= 2 && strcmp(argv[1], "host") == 0)
        return host_checks();
    if (argc >= 4 && strcmp(argv[1], "gpu") == 0)
        return gpu_step(argv[2], argv[3]);
    fprintf(stderr, "usage: %s host | gpu <in.bin> <out.bin>\n", argv[0]);
    return 2;
}
