/*
 * CPU oracle for the Ulysses 4D all-to-all re-layout.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg use it. It shares no code, header or constant with the CUDA library.
 *
 * What it computes (the plain definition, per element, nested loops):
 *
 *   FastVideo API docs, device_communicators/ulysses_a2a, `run_armed`:
 *   mode 0 takes each rank's [B, S_local, H, D] to [B, S_local*w, H/w, D]
 *   (heads scattered, sequence gathered); any other mode takes
 *   [B, S_local*w, H/w, D] back to [B, S_local, H, D]. The native op is always
 *   handed the mode-0-local tuple (B, S_local, H, D) in both modes.
 *
 *   The element map (the standard Ulysses ordering: rank r keeps head group r,
 *   the gathered sequence is rank-major):
 *     mode 0:  out_r[b, j*S_local + s, h', d] = x_j[b, s, r*(H/w) + h', d]
 *     mode 1:  out_j[b, s, r*(H/w) + h', d]   = x_r[b, j*S_local + s, h', d]
 *   for r, j in [0, w), b in [0, B), s in [0, S_local), h' in [0, H/w),
 *   d in [0, D). Mode 1 is the exact inverse of mode 0.
 *
 *   Chunked variant (same page, `run_armed`, `chunked` branch): for each plane
 *   b, the same op runs on the one-plane views x[b:b+1], out[b:b+1] with B = 1.
 *
 * Elements are copied as raw bytes (elem_bytes each): no arithmetic touches a
 * value, so NaN payloads and signed zeros survive unchanged.
 *
 * Two builds of this one file: the plain single-threaded one, and an OpenMP
 * one (gcc -fopenmp) that splits the outermost (r, b) loop pair over the host
 * cores. Each (r, b) iteration writes its own disjoint part of the outputs
 * (mode 0: plane b of out_r; mode 1: head group r of plane b of every out_j),
 * so the split changes only the order in which elements are copied, never a
 * result. Without -fopenmp the pragmas are compiled out.
 *
 * Return codes: 0 = done; -1 = bad argument (null pointer for a non-empty
 * slab, negative size, H not divisible by w, unsupported mode or element
 * size). Zero sizes are an empty re-layout: done, nothing touched.
 */
#include <stdint.h>
#include <string.h>

/* The (r, b) loop pair is split over threads in the OpenMP build only. */
#ifdef _OPENMP
#define OUTER_LOOPS_PARALLEL _Pragma("omp parallel for collapse(2) schedule(static)")
#else
#define OUTER_LOOPS_PARALLEL
#endif

/* A size of 0 makes the index set empty: nothing is read or written, and
 * the slab pointers may then be NULL. */
static int bad_args(const void *const *in, void *const *out, int64_t B,
                    int64_t S_local, int64_t H, int64_t D, int w, int mode,
                    int elem_bytes)
{
    if (in == NULL || out == NULL) return 1;
    if (w < 1 || B < 0 || S_local < 0 || H < 0 || D < 0) return 1;
    if (H % w != 0) return 1;
    if (mode != 0 && mode != 1) return 1;
    if (elem_bytes < 1) return 1;
    const int empty = (B == 0 || S_local == 0 || H == 0 || D == 0);
    for (int k = 0; k < w && !empty; ++k)
        if (in[k] == NULL || out[k] == NULL) return 1;
    return 0;
}

/* Offset (in elements) of [b, s, h, d] in a row-major [*, S, Hn, D] tensor. */
static int64_t at4(int64_t b, int64_t s, int64_t h, int64_t d,
                   int64_t S, int64_t Hn, int64_t D)
{
    return ((b * S + s) * Hn + h) * D + d;
}

int oracle_ulysses_a2a(const void *const *in, void *const *out, int64_t B,
                       int64_t S_local, int64_t H, int64_t D, int w, int mode,
                       int elem_bytes)
{
    if (bad_args(in, out, B, S_local, H, D, w, mode, elem_bytes)) return -1;
    const int64_t Hw = H / w;          /* heads per rank after the scatter */
    const int64_t S_global = S_local * w;
    const int64_t E = elem_bytes;

    OUTER_LOOPS_PARALLEL
    for (int64_t r = 0; r < w; ++r)
        for (int64_t b = 0; b < B; ++b)
            for (int j = 0; j < w; ++j)
                for (int64_t s = 0; s < S_local; ++s)
                    for (int64_t hp = 0; hp < Hw; ++hp)
                        for (int64_t d = 0; d < D; ++d) {
                            /* the two sides of the same correspondence */
                            /* A: rank j's sequence shard, all H heads    */
                            int64_t a = at4(b, s, r * Hw + hp, d,
                                            S_local, H, D);
                            /* C: rank r's head group, whole sequence    */
                            int64_t c = at4(b, (int64_t)j * S_local + s, hp, d,
                                            S_global, Hw, D);
                            if (mode == 0) {
                                /* out_r[b, j*S_local+s, h', d] = x_j[b, s, r*Hw+h', d] */
                                const char *src = (const char *)in[j] + a * E;
                                char *dst = (char *)out[r] + c * E;
                                memcpy(dst, src, (size_t)E);
                            } else {
                                /* out_j[b, s, r*Hw+h', d] = x_r[b, j*S_local+s, h', d] */
                                const char *src = (const char *)in[r] + c * E;
                                char *dst = (char *)out[j] + a * E;
                                memcpy(dst, src, (size_t)E);
                            }
                        }
    return 0;
}

/* Same map with the [B, S_local, H, D] side laid out with a row pitch: the
 * element (b, s, h, d) of that side sits at ((b*S_local + s)*row_pitch + h*D + d)
 * (row_pitch >= H*D elements; the gathered side stays dense). This is the
 * layout of, e.g., q inside a packed [B, S_local, 3, H, D] projection output
 * (row_pitch = 3*H*D). Elements in the gap between H*D and row_pitch are
 * neither read nor written. */
int oracle_ulysses_a2a_pitched(const void *const *in, void *const *out,
                               int64_t B, int64_t S_local, int64_t H, int64_t D,
                               int w, int mode, int elem_bytes, int64_t row_pitch)
{
    if (bad_args(in, out, B, S_local, H, D, w, mode, elem_bytes)) return -1;
    if (row_pitch < H * D) return -1;
    const int64_t Hw = H / w;
    const int64_t S_global = S_local * w;
    const int64_t E = elem_bytes;
    OUTER_LOOPS_PARALLEL
    for (int64_t r = 0; r < w; ++r)
        for (int64_t b = 0; b < B; ++b)
            for (int j = 0; j < w; ++j)
                for (int64_t s = 0; s < S_local; ++s)
                    for (int64_t hp = 0; hp < Hw; ++hp)
                        for (int64_t d = 0; d < D; ++d) {
                            /* pitched side: rank j's row (b, s), head r*Hw + h' */
                            int64_t a = (b * S_local + s) * row_pitch
                                        + (r * Hw + hp) * D + d;
                            int64_t c = at4(b, (int64_t)j * S_local + s, hp, d,
                                            S_global, Hw, D);
                            if (mode == 0) {
                                const char *src = (const char *)in[j] + a * E;
                                char *dst = (char *)out[r] + c * E;
                                memcpy(dst, src, (size_t)E);
                            } else {
                                const char *src = (const char *)in[r] + c * E;
                                char *dst = (char *)out[j] + a * E;
                                memcpy(dst, src, (size_t)E);
                            }
                        }
    return 0;
}

/* The chunked variant: one call per plane, each on B = 1 plane views. */
int oracle_ulysses_a2a_chunked(const void *const *in, void *const *out,
                               int64_t B, int64_t S_local, int64_t H, int64_t D,
                               int w, int mode, int elem_bytes)
{
    if (bad_args(in, out, B, S_local, H, D, w, mode, elem_bytes)) return -1;
    if (w > 1024) return -1;
    const int64_t E = elem_bytes;
    /* elements in one plane of a [B, S_local, H, D] slab; the other layout,
       [B, S_local*w, H/w, D], holds the same count per plane */
    const int64_t plane = S_local * H * D;
    const void *in_v[1024];
    void *out_v[1024];
    for (int64_t b = 0; b < B; ++b) {
        for (int k = 0; k < w; ++k) {
            in_v[k] = (const char *)in[k] + b * plane * E;
            out_v[k] = (char *)out[k] + b * plane * E;
        }
        int rc = oracle_ulysses_a2a(in_v, out_v, 1, S_local, H, D, w, mode,
                                    elem_bytes);
        if (rc != 0) return rc;
    }
    return 0;
}
