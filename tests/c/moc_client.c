/* A plain C99 client of the MoC library: the forward pass driven through the
 * C ABI alone (include/moc.h + libmoc.so + the CUDA runtime for device
 * memory), with no Python or C++ in between.
 *
 *   moc_client --host-only
 *       builds a host-only layout of a small scene and checks the calls that
 *       need no GPU: layout sizes, status strings, argument rejection.
 *   moc_client IN OUT
 *       reads a scene and its inputs from IN, runs (1) pooling, (2) routing and
 *       the attention stage on device 0, and writes O, lse and sel to OUT.
 *
 * IN (little-endian): int32 magic 0x4d6f4331, n_segments, anchor_mode,
 * local_radius, B, H, d, k, causal; int32 seg_len[n], seg_kind[n],
 * seg_shot[n], seg_frame[n]; then Q, K, V as bf16 [B][H][L][d].
 * OUT: O bf16 [B][H][L][d], lse fp32 [B][H][L], sel int32 [B][H][L][k].
 * Exit status 0 on success; a message on stderr otherwise. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "moc.h"

#define FAIL(...) do { fprintf(stderr, __VA_ARGS__); fputc('\n', stderr); return 1; } while (0)

static int host_only(void) {
    /* 8 caption tokens, then 2 shots x 2 frames of 16 tokens */
    const int32_t len[5] = {8, 16, 16, 16, 16}, kind[5] = {MOC_CAPTION, MOC_VIDEO, MOC_VIDEO, MOC_VIDEO, MOC_VIDEO};
    const int32_t shot[5] = {0, 0, 0, 1, 1}, frame[5] = {-1, 0, 1, 0, 1};
    moc_layout_desc desc;
    moc_layout* lay = NULL;
    int64_t L = 0;
    int32_t C = 0, S = 0;
    int32_t bad_len[5];
    char dummy[256];
    desc.n_segments = 5;
    desc.seg_len = len;
    desc.seg_kind = kind;
    desc.seg_shot = shot;
    desc.seg_frame = frame;
    desc.anchor_mode = MOC_ANCHOR_SHOT;
    desc.local_radius = 0;
    if (moc_build_layout(&desc, -1, &lay) != MOC_OK || !lay) FAIL("host-only layout not built");
    if (moc_layout_info(lay, &L, &C, &S) != MOC_OK || L != 72 || C != 5 || S != 2)
        FAIL("layout info: L=%lld C=%d shots=%d", (long long)L, C, S);
    if (strlen(moc_status_string(MOC_OK)) == 0 || strlen(moc_status_string(MOC_ERR_LAYOUT)) == 0)
        FAIL("empty status string");
    /* compute calls reject a host-only layout before touching memory */
    if (moc_pool_keys(lay, 1, 1, 64, dummy, (float*)dummy, NULL) != MOC_ERR_INVALID_ARG)
        FAIL("pool on a host-only layout was not rejected");
    moc_layout_destroy(lay);
    /* an empty chunk is a bad layout, and *out is cleared */
    memcpy(bad_len, len, sizeof bad_len);
    bad_len[2] = 0;
    desc.seg_len = bad_len;
    lay = (moc_layout*)dummy;
    if (moc_build_layout(&desc, -1, &lay) != MOC_ERR_LAYOUT || lay != NULL) FAIL("empty chunk accepted");
    printf("ok\n");
    return 0;
}

static int read_i32(FILE* f, int32_t* v, size_t n) { return fread(v, sizeof(int32_t), n, f) == n; }

static int device_run(const char* in_path, const char* out_path) {
    FILE* f = fopen(in_path, "rb");
    int32_t hdr[9], n, B, H, d, k, causal;
    int32_t *len = NULL, *kind = NULL, *shot = NULL, *frame = NULL;
    moc_layout_desc desc;
    moc_layout* lay = NULL;
    int64_t L = 0;
    int32_t C = 0;
    size_t nqkv, ws_bytes;
    uint16_t* host = NULL;
    void *dQ = NULL, *dK = NULL, *dV = NULL, *dO = NULL, *ws = NULL;
    float *dKbar = NULL, *dlse = NULL, *lse = NULL;
    int32_t *dsel = NULL, *sel = NULL, detail = 0;
    moc_status st;
    int rc = 1;
    if (!f) FAIL("cannot open %s", in_path);
    if (!read_i32(f, hdr, 9) || hdr[0] != 0x4d6f4331) FAIL("bad input header");
    n = hdr[1]; B = hdr[4]; H = hdr[5]; d = hdr[6]; k = hdr[7]; causal = hdr[8];
    len = malloc(4 * (size_t)n); kind = malloc(4 * (size_t)n);
    shot = malloc(4 * (size_t)n); frame = malloc(4 * (size_t)n);
    if (!read_i32(f, len, n) || !read_i32(f, kind, n) || !read_i32(f, shot, n) || !read_i32(f, frame, n))
        FAIL("short segment tables");
    desc.n_segments = n;
    desc.seg_len = len;
    desc.seg_kind = kind;
    desc.seg_shot = shot;
    desc.seg_frame = frame;
    desc.anchor_mode = hdr[2];
    desc.local_radius = hdr[3];
    if (cudaSetDevice(0) != cudaSuccess) FAIL("no CUDA device");
    if ((st = moc_build_layout(&desc, 0, &lay)) != MOC_OK) FAIL("layout: %s", moc_status_string(st));
    moc_layout_info(lay, &L, &C, NULL);
    nqkv = (size_t)B * H * (size_t)L * d;
    host = malloc(3 * nqkv * 2);
    if (fread(host, 2, 3 * nqkv, f) != 3 * nqkv) FAIL("short Q/K/V");
    fclose(f);
    ws_bytes = moc_attention_workspace_bytes(lay, B, H, d, k);
    if (cudaMalloc(&dQ, nqkv * 2) || cudaMalloc(&dK, nqkv * 2) || cudaMalloc(&dV, nqkv * 2) ||
        cudaMalloc(&dO, nqkv * 2) || cudaMalloc((void**)&dKbar, (size_t)B * H * C * d * 4) ||
        cudaMalloc((void**)&dlse, (size_t)B * H * L * 4) ||
        cudaMalloc((void**)&dsel, (size_t)B * H * L * (k > 0 ? k : 1) * 4) || cudaMalloc(&ws, ws_bytes))
        FAIL("cudaMalloc");
    if (cudaMemcpy(dQ, host, nqkv * 2, cudaMemcpyHostToDevice) ||
        cudaMemcpy(dK, host + nqkv, nqkv * 2, cudaMemcpyHostToDevice) ||
        cudaMemcpy(dV, host + 2 * nqkv, nqkv * 2, cudaMemcpyHostToDevice))
        FAIL("upload");
    /* (1) pool, (2) route, then (3)-(5) on the default stream */
    if ((st = moc_pool_keys(lay, B, H, d, dK, dKbar, NULL)) != MOC_OK) FAIL("pool: %s", moc_status_string(st));
    if (k > 0 && (st = moc_route(lay, B, H, d, dQ, dKbar, k, causal, dsel, NULL)) != MOC_OK)
        FAIL("route: %s", moc_status_string(st));
    st = moc_attention_fwd(lay, B, H, d, dQ, dK, dV, k > 0 ? dsel : NULL, k, 1.0f / sqrtf((float)d), dO,
                           dlse, ws, ws_bytes, NULL);
    if (st != MOC_OK) FAIL("attention: %s", moc_status_string(st));
    if ((st = moc_check_device_error(ws, ws_bytes, &detail, NULL)) != MOC_OK)
        FAIL("device error word: %s (%d)", moc_status_string(st), detail);
    if ((st = moc_layout_device_error(lay, &detail, NULL)) != MOC_OK)
        FAIL("router error word: %s (%d)", moc_status_string(st), detail);
    lse = malloc((size_t)B * H * L * 4);
    sel = malloc((size_t)B * H * L * (k > 0 ? k : 1) * 4);
    if (cudaMemcpy(host, dO, nqkv * 2, cudaMemcpyDeviceToHost) ||
        cudaMemcpy(lse, dlse, (size_t)B * H * L * 4, cudaMemcpyDeviceToHost) ||
        (k > 0 && cudaMemcpy(sel, dsel, (size_t)B * H * L * k * 4, cudaMemcpyDeviceToHost)))
        FAIL("download");
    f = fopen(out_path, "wb");
    if (!f) FAIL("cannot write %s", out_path);
    if (fwrite(host, 2, nqkv, f) == nqkv && fwrite(lse, 4, (size_t)B * H * L, f) == (size_t)B * H * L &&
        (k == 0 || fwrite(sel, 4, (size_t)B * H * L * k, f) == (size_t)B * H * L * k))
        rc = 0;
    fclose(f);
    cudaFree(dQ); cudaFree(dK); cudaFree(dV); cudaFree(dO); cudaFree(dKbar); cudaFree(dlse);
    cudaFree(dsel); cudaFree(ws);
    moc_layout_destroy(lay);
    free(len); free(kind); free(shot); free(frame); free(host); free(lse); free(sel);
    if (rc) FAIL("short write");
    return 0;
}

int main(int argc, char** argv) {
    if (argc == 2 && strcmp(argv[1], "--host-only") == 0) return host_only();
    if (argc == 3) return device_run(argv[1], argv[2]);
    fprintf(stderr, "usage: %s --host-only | %s IN OUT\n", argv[0], argv[0]);
    return 2;
}
