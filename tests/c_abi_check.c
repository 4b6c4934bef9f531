/*
 * Plain-C user of libulysses_a2a.so (no Python, no torch): allocates rank
 * slabs with cudaMalloc, runs both modes through ulysses_a2a_run, runs the
 * host-buffer entry point, checks the error codes of a few rejected calls, runs
 * the multi-GPU exchange entry points with its ranks in this process, runs a
 * head-packed launch (three tensors, one call of ulysses_a2a_run_ex), and
 * compares every output byte with the CPU oracle (libulysses_oracle.so, test
 * infrastructure). Exit status 0 = all checks passed.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "ulysses_a2a.h"

int oracle_ulysses_a2a(const void *const *in, void *const *out, int64_t B,
                       int64_t S_local, int64_t H, int64_t D, int w, int mode,
                       int elem_bytes);
int oracle_ulysses_a2a_pitched(const void *const *in, void *const *out,
                               int64_t B, int64_t S_local, int64_t H, int64_t D,
                               int w, int mode, int elem_bytes, int64_t row_pitch);

#define W 4
#define CHECK(cond, msg)                                             \
    do {                                                             \
        if (!(cond)) {                                               \
            fprintf(stderr, "FAILED: %s (line %d)\n", msg, __LINE__); \
            return 1;                                                \
        }                                                            \
    } while (0)

int main(void) {
    const int64_t B = 2, S = 37, H = 8, D = 64;
    const int E = 2;
    const size_t n = (size_t)(B * S * H * D);
    const size_t bytes = n * E;
    uint16_t *hin[W], *hout[W], *want[W], *hback[W];
    void *din[W], *dout[W];
    for (int k = 0; k < W; ++k) {
        hin[k] = malloc(bytes);
        hout[k] = malloc(bytes);
        want[k] = malloc(bytes);
        hback[k] = malloc(bytes);
        for (size_t i = 0; i < n; ++i) hin[k][i] = (uint16_t)(k * 40503u + i * 2654435761u);
        CHECK(cudaMalloc(&din[k], bytes) == cudaSuccess, "cudaMalloc in");
        CHECK(cudaMalloc(&dout[k], bytes) == cudaSuccess, "cudaMalloc out");
        CHECK(cudaMemcpy(din[k], hin[k], bytes, cudaMemcpyHostToDevice) == cudaSuccess, "H2D");
    }
    ulysses_a2a_ctx *ctx = NULL;
    CHECK(ulysses_a2a_create(&ctx, 0, E) == ULYSSES_A2A_OK && ctx != NULL, "create");

    /* mode 0 on device slabs, against the oracle */
    CHECK(oracle_ulysses_a2a((const void *const *)hin, (void *const *)want, B, S, H, D, W, 0, E) == 0,
          "oracle mode 0");
    CHECK(ulysses_a2a_run(ctx, (const void *const *)din, dout, B, S, H, D, W, 0, 0, NULL) ==
              ULYSSES_A2A_OK, ulysses_a2a_last_error(ctx));
    CHECK(ulysses_a2a_status(ctx, NULL) == ULYSSES_A2A_OK, "status after mode 0");
    for (int k = 0; k < W; ++k) {
        CHECK(cudaMemcpy(hout[k], dout[k], bytes, cudaMemcpyDeviceToHost) == cudaSuccess, "D2H");
        CHECK(memcmp(hout[k], want[k], bytes) == 0, "mode 0 differs from the oracle");
    }
    /* mode 1 (chunked per plane) back into the inputs' layout: the round trip */
    CHECK(ulysses_a2a_run(ctx, (const void *const *)dout, din, B, S, H, D, W, 1, 1, NULL) ==
              ULYSSES_A2A_OK, ulysses_a2a_last_error(ctx));
    for (int k = 0; k < W; ++k) {
        CHECK(cudaMemcpy(hback[k], din[k], bytes, cudaMemcpyDeviceToHost) == cudaSuccess, "D2H");
        CHECK(memcmp(hback[k], hin[k], bytes) == 0, "mode 1 did not undo mode 0");
    }
    /* the host-buffer entry point */
    for (int k = 0; k < W; ++k) memset(hout[k], 0xFF, bytes);
    CHECK(ulysses_a2a_run_host(ctx, (const void *const *)hin, (void *const *)hout, B, S, H, D, W, 0,
                               0, NULL) == ULYSSES_A2A_OK, ulysses_a2a_last_error(ctx));
    for (int k = 0; k < W; ++k) CHECK(memcmp(hout[k], want[k], bytes) == 0, "run_host differs");

    /* rejected calls launch nothing and leave the context usable */
    const uint64_t launches = ulysses_a2a_launch_count(ctx);
    CHECK(ulysses_a2a_run(ctx, (const void *const *)din, dout, B, S, 7, D, W, 0, 0, NULL) ==
              ULYSSES_A2A_ERR_INVALID, "H % w accepted");
    void *alias[W] = {din[0], dout[1], dout[2], dout[3]};
    CHECK(ulysses_a2a_run(ctx, (const void *const *)din, alias, B, S, H, D, W, 0, 0, NULL) ==
              ULYSSES_A2A_ERR_OVERLAP, "overlap accepted");
    void *host_ptrs[W] = {hout[0], hout[1], hout[2], hout[3]};
    CHECK(ulysses_a2a_run(ctx, (const void *const *)din, host_ptrs, B, S, H, D, W, 0, 0, NULL) ==
              ULYSSES_A2A_ERR_DEVICE, "host pointer accepted as device memory");
    CHECK(ulysses_a2a_launch_count(ctx) == launches, "a rejected call launched work");
    CHECK(strlen(ulysses_a2a_last_error(ctx)) > 0, "no error message");

    /* the multi-GPU exchange with its W ranks in this process: one context and
       window per rank, records handed over in memory; every publish, then every
       pull, on the default stream (stream order stands in for the barriers) */
    {
        ulysses_a2a_ctx *rctx[W];
        ulysses_a2a_peer *peer[W];
        unsigned char rec[W][ULYSSES_A2A_PEER_HANDLE_BYTES];
        for (int k = 0; k < W; ++k) {
            CHECK(ulysses_a2a_create(&rctx[k], 0, E) == ULYSSES_A2A_OK, "create (rank)");
            CHECK(ulysses_a2a_peer_create(rctx[k], k, W, bytes, &peer[k], rec[k]) ==
                      ULYSSES_A2A_OK, ulysses_a2a_last_error(rctx[k]));
        }
        for (int k = 0; k < W; ++k)
            CHECK(ulysses_a2a_peer_open(peer[k], rec) == ULYSSES_A2A_OK,
                  ulysses_a2a_last_error(rctx[k]));
        CHECK(ulysses_a2a_peer_window_bytes(peer[0]) == bytes, "window size");
        for (int k = 0; k < W; ++k) {
            CHECK(cudaMemcpy(din[k], hin[k], bytes, cudaMemcpyHostToDevice) == cudaSuccess, "H2D");
            CHECK(cudaMemset(dout[k], 0xFF, bytes) == cudaSuccess, "poison");
        }
        for (int k = 0; k < W; ++k)
            CHECK(ulysses_a2a_peer_publish(peer[k], din[k], B, S, H, D, 0, 0, 0, NULL) ==
                      ULYSSES_A2A_OK, ulysses_a2a_last_error(rctx[k]));
        for (int k = 0; k < W; ++k)
            CHECK(ulysses_a2a_peer_pull(peer[k], dout[k], B, S, H, D, 0, 0, 0, NULL) ==
                      ULYSSES_A2A_OK, ulysses_a2a_last_error(rctx[k]));
        for (int k = 0; k < W; ++k) {
            CHECK(cudaMemcpy(hout[k], dout[k], bytes, cudaMemcpyDeviceToHost) == cudaSuccess, "D2H");
            CHECK(memcmp(hout[k], want[k], bytes) == 0, "peer exchange differs from the oracle");
        }
        for (int k = 0; k < W; ++k) CHECK(ulysses_a2a_peer_close(peer[k]) == ULYSSES_A2A_OK, "close");
        for (int k = 0; k < W; ++k) {
            CHECK(ulysses_a2a_peer_destroy(peer[k]) == ULYSSES_A2A_OK, "peer destroy");
            CHECK(ulysses_a2a_destroy(rctx[k]) == ULYSSES_A2A_OK, "destroy (rank)");
        }
        CHECK(ulysses_a2a_peer_destroy(NULL) == ULYSSES_A2A_OK, "peer destroy(NULL)");
    }

    /* three head-packed tensors in one launch: in[j] is [B, S, 3, H, D], out[t*W + r]
       tensor t's [B, S*W, H/W, D] slab of rank r; the oracle runs once per tensor
       on the row-pitched views (pitch 3*H*D, offset t*H*D) */
    {
        enum { T = 3 };
        const size_t pn = n * T, pbytes = pn * E;
        uint16_t *hp[W], *hq[T * W], *wq[T * W];
        void *dp[W], *dq[T * W];
        for (int k = 0; k < W; ++k) {
            hp[k] = malloc(pbytes);
            for (size_t i = 0; i < pn; ++i) hp[k][i] = (uint16_t)(k * 7919u + i * 40503u);
            CHECK(cudaMalloc(&dp[k], pbytes) == cudaSuccess, "cudaMalloc packed");
            CHECK(cudaMemcpy(dp[k], hp[k], pbytes, cudaMemcpyHostToDevice) == cudaSuccess, "H2D");
        }
        for (int k = 0; k < T * W; ++k) {
            hq[k] = malloc(bytes);
            wq[k] = malloc(bytes);
            CHECK(cudaMalloc(&dq[k], bytes) == cudaSuccess, "cudaMalloc gathered");
        }
        for (int t = 0; t < T; ++t) {
            const void *views[W];
            void *wants[W];
            for (int k = 0; k < W; ++k) {
                views[k] = hp[k] + (size_t)t * H * D;
                wants[k] = wq[t * W + k];
            }
            CHECK(oracle_ulysses_a2a_pitched(views, wants, B, S, H, D, W, 0, E, T * H * D) == 0,
                  "pitched oracle");
        }
        ulysses_a2a_desc_t d;
        memset(&d, 0, sizeof(d));
        d.in_slabs = (const void *const *)dp;
        d.out_slabs = dq;
        d.B = B; d.S_local = S; d.H = H; d.D = D;
        d.w = W; d.mode = 0; d.chunked = 0; d.ntensors = T; d.row_pitch = 0;
        const uint64_t l0 = ulysses_a2a_launch_count(ctx);
        CHECK(ulysses_a2a_run_ex(ctx, &d, NULL) == ULYSSES_A2A_OK, ulysses_a2a_last_error(ctx));
        CHECK(ulysses_a2a_launch_count(ctx) == l0 + 1, "packed call is one launch");
        for (int k = 0; k < T * W; ++k) {
            CHECK(cudaMemcpy(hq[k], dq[k], bytes, cudaMemcpyDeviceToHost) == cudaSuccess, "D2H");
            CHECK(memcmp(hq[k], wq[k], bytes) == 0, "packed launch differs from the oracle");
        }
        for (int k = 0; k < W; ++k) { cudaFree(dp[k]); free(hp[k]); }
        for (int k = 0; k < T * W; ++k) { cudaFree(dq[k]); free(hq[k]); free(wq[k]); }
    }

    CHECK(ulysses_a2a_destroy(ctx) == ULYSSES_A2A_OK, "destroy");
    CHECK(ulysses_a2a_destroy(NULL) == ULYSSES_A2A_OK, "destroy(NULL)");
    for (int k = 0; k < W; ++k) {
        cudaFree(din[k]);
        cudaFree(dout[k]);
        free(hin[k]);
        free(hout[k]);
        free(want[k]);
        free(hback[k]);
    }
    printf("c_abi_check: all checks passed\n");
    return 0;
}
