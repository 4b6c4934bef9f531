/*
 * ulysses_a2a.h - C ABI of the B200 Ulysses 4D all-to-all re-layout library
 * (libulysses_a2a.so).
 *
 * The operation (FastVideo API docs, fastvideo.distributed.device_communicators
 * .ulysses_a2a, `run_armed`): Ulysses sequence parallelism keeps, on each of w
 * ranks, a sequence shard x_r of shape [B, S_local, H, D]. Before attention,
 * "mode 0" scatters heads and gathers sequence, so that every rank holds the
 * whole sequence for H/w heads, [B, S_local*w, H/w, D]; after attention "mode 1"
 * undoes it. Here all w rank slabs live in one GPU's memory, so the all-to-all
 * is a pure permutation of bytes:
 *
 *   mode 0:  out_r[b, j*S_local + s, h', d] = x_j[b, s, r*(H/w) + h', d]
 *   mode 1:  out_j[b, s, r*(H/w) + h', d]   = x_r[b, j*S_local + s, h', d]
 *
 * for ranks r, j in [0, w), b in [0, B), s in [0, S_local), h' in [0, H/w),
 * d in [0, D). Rank r receives head group [r*H/w, (r+1)*H/w); the gathered
 * sequence is rank-major. Values are moved as raw elem_bytes-byte words: no
 * arithmetic, bit-exact, NaN payloads and -0.0 preserved.
 *
 * Layout: every slab is a dense row-major C array. In mode 0 each in_slabs[j]
 * is [B, S_local, H, D] and each out_slabs[r] is [B, S_local*w, H/w, D]; in
 * mode 1 the roles are swapped. (B, S_local, H, D) are ALWAYS passed in
 * mode-0-local terms, whichever the mode, as the page's native op receives them.
 * ulysses_a2a_run_ex adds row-pitched slabs and head-packed tensors (several
 * tensors in one launch); the ulysses_a2a_peer_* functions run the same map
 * across GPUs, one process per GPU.
 *
 * Ownership: the caller owns every slab and the stream. The context owns a tiny
 * device status word, a cache of TMA descriptors, and two device buffers that
 * exist only once they are used and then grow on demand: the staging window of
 * chunked = 2 calls (one plane of every input slab) and the staging buffers of
 * ulysses_a2a_run_host. A peer object owns its rank's window. Nothing returned
 * by this API ever aliases caller memory.
 *
 * Launches: every kernel is launched with programmatic stream serialization
 * (programmatic dependent launch) and waits for the previous grid in the
 * stream (griddepcontrol.wait) before it touches memory, so it is safe after
 * any producer. It also signals its dependents early: a kernel the caller
 * launches next on the same stream WITH programmatic stream serialization
 * must call cudaGridDependencySynchronize() before reading these outputs, as
 * the CUDA programming model requires of such kernels. Kernels launched
 * without that attribute, copies and events see the usual stream order.
 *
 * Errors: every entry point returns an int status (ULYSSES_A2A_OK = 0). All
 * arguments are checked on the host BEFORE anything is launched; a rejected
 * call launches nothing, leaves the outputs untouched and the context usable,
 * and ulysses_a2a_last_error() describes why. Misalignment is not an error: it
 * only selects a narrower copy path. Thread safety: one context must not be
 * used from two host threads at once; distinct contexts are independent.
 */
#ifndef ULYSSES_A2A_H
#define ULYSSES_A2A_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define ULYSSES_A2A_OK              0
#define ULYSSES_A2A_ERR_INVALID     1  /* bad argument: null, size, H % w, mode */
#define ULYSSES_A2A_ERR_OVERLAP     2  /* an output slab overlaps another slab  */
#define ULYSSES_A2A_ERR_DEVICE      3  /* pointer not in ctx's device memory, or
                                          its allocation is smaller than the slab */
#define ULYSSES_A2A_ERR_CUDA        4  /* a CUDA runtime/driver call failed     */
#define ULYSSES_A2A_ERR_UNSUPPORTED 5  /* forced path cannot express the shape  */
#define ULYSSES_A2A_ERR_NOMEM       6  /* host or device allocation failed      */
#define ULYSSES_A2A_ERR_TIMEOUT     7  /* a kernel's bounded wait gave up       */
#define ULYSSES_A2A_ERR_INTERNAL    8  /* an unexpected host-side failure inside
                                          the library (no exception ever leaves
                                          an entry point)                       */

/* ---- copy paths ------------------------------------------------------- */
#define ULYSSES_A2A_PATH_AUTO 0  /* TMA when the shape allows it; else VEC, or
                                    STAGED when VEC could only use vectors
                                    of 4 bytes or less and cannot peel them
                                    (see plan_t.peeled), or 8-byte vectors
                                    that the staged path's fixed-phase form
                                    takes                                   */
#define ULYSSES_A2A_PATH_TMA  1  /* cp.async.bulk.tensor load -> smem -> store */
#define ULYSSES_A2A_PATH_VEC  2  /* 16/8/4/2/1-byte LDG/STG copy, or 16-byte
                                    vectors between peeled heads and tails
                                    (plan_t.peeled)                          */
#define ULYSSES_A2A_PATH_STAGED 3 /* 16-byte LDG/STG, re-aligned in shared
                                    memory: runs or bases off 16 bytes     */

#define ULYSSES_A2A_MAX_W     64 /* largest rank count any path accepts        */
#define ULYSSES_A2A_CHUNKED_WINDOW 2 /* chunked = 2: per plane via a window   */
#define ULYSSES_A2A_MAX_W_TMA 8  /* largest rank count of the TMA path         */

typedef struct ulysses_a2a_ctx ulysses_a2a_ctx; /* opaque */

/* Geometry and path the library picks for one call (see ulysses_a2a_plan). */
typedef struct ulysses_a2a_plan_t {
    int32_t path;            /* ULYSSES_A2A_PATH_TMA, _VEC or _STAGED         */
    int32_t vec_bytes;       /* VEC path: bytes per load/store (16..1);
                                STAGED: bytes per piece re-aligned in shared
                                memory (global accesses are 16 bytes)       */
    int64_t row_bytes;       /* one contiguous run: (H/w)*D*elem_bytes        */
    int64_t rows_per_tile;   /* S_tile: sequence rows per work unit           */
    int64_t tiles_per_block; /* ceil(S_local / S_tile)                        */
    int64_t tail_rows;       /* S_local % S_tile (0 = no ragged tile)         */
    int64_t units;           /* work units per launch: w * B_launch * w * T
                                (STAGED: w * B_launch * T, each unit moving
                                every head group of its rows)              */
    int64_t payload_bytes;   /* sum of input slab bytes = w*B*S_local*H*D*E   */
    int32_t launches;        /* kernel launches per call: 1, or B if chunked  */
    int32_t grid;            /* CTAs per launch                               */
    int32_t block;           /* threads per CTA                               */
    int32_t stages;          /* TMA path: shared-memory tiles per CTA (all
                                producers together)                        */
    int32_t lookahead;       /* TMA path: loads in flight per producer       */
    int32_t producers;       /* TMA path: producer warps per CTA (1..8)      */
    int64_t smem_bytes;      /* dynamic shared memory per CTA                 */
    int32_t order;           /* unit numbering: 0 = destination rank r
                                outermost, 1 = r innermost                  */
    int32_t chunk_units;     /* TMA path: 0 = persistent grid (static round
                                robin); n = n consecutive units per CTA     */
    int64_t row_pitch;       /* elements between rows of the [B,S_local,H,D]
                                side (H*D when dense)                       */
    int32_t peeled;          /* VEC path, runs and rows multiples of 16
                                bytes, runs of 64+: 1 = every slab starts the
                                same a bytes past a 16-byte boundary; each run
                                moves as 16-byte vectors between a head of
                                16 - a and a tail of a bytes, moved in aligned
                                pieces by the same CTAs. 2 = the input slabs
                                share one offset and the output slabs another:
                                each destination vector (and head and tail) is
                                two aligned source vectors joined by a shift.
                                vec_bytes is then 16                        */
    int32_t fixed_phase;     /* STAGED path: 1 = the [B,S_local,H,D] side is
                                dense and the gathered slabs share one
                                offset past a 16-byte boundary: each thread
                                takes chunks that share one offset modulo a
                                strided row (or, for mode 0 with pieces of
                                4 or 8 bytes, gathered chunks that share one
                                offset modulo a run, built from an image of
                                the strided rows), so it works out where
                                their pieces go once per work unit; 0 = every
                                chunk's pieces are placed one by one        */
} ulysses_a2a_plan_t;

/* One call's arguments, for ulysses_a2a_run_ex / ulysses_a2a_plan_ex. Same
 * meaning as the ulysses_a2a_run parameters, plus:
 *
 * row_pitch: the number of elements between consecutive (b, s) rows of the
 * [B, S_local, H, D] side (the inputs in mode 0, the outputs in mode 1), whose
 * planes are then S_local*row_pitch elements apart; 0 means dense. A pitch
 * > H*D lets mode 0 read q, k or v in place from a packed [B, S_local, 3, H, D]
 * projection output (row_pitch = 3*H*D, slab pointers offset by 0, H*D or
 * 2*H*D elements), and lets mode 1 write into such a packed buffer; elements
 * between H*D and row_pitch are neither read nor written. The other side is
 * always dense.
 *
 * ntensors: 0 or 1 for one tensor per rank. T > 1 re-lays out T tensors packed
 * along the head dimension in one launch (for example q, k and v of a
 * [B, S_local, 3, H, D] projection output): the [B, S_local, T, H, D] side has
 * w slabs (rows of T*H*D elements, or row_pitch), the other side T*w dense
 * [B, S_local*w, H/w, D] slabs ordered tensor-major, slab t*w + r being
 * tensor t's slab of rank r:
 *   mode 0: out[t*w + r][b, j*S_local + s, h', d] = in[j][b, s, t, r*(H/w) + h', d]
 *   mode 1: out[j][b, s, t, r*(H/w) + h', d]     = in[t*w + r][b, j*S_local + s, h', d]
 * Equal to T separate calls on the row-pitched views of each tensor. Needs
 * T*w <= ULYSSES_A2A_MAX_W and chunked 0 or 1; uses the VEC path. */
typedef struct ulysses_a2a_desc_t {
    const void *const *in_slabs;
    void *const *out_slabs;
    int64_t B, S_local, H, D;
    int32_t w, mode, chunked;
    int32_t ntensors;        /* 0 or 1: one tensor; T > 1: head-packed tensors */
    int64_t row_pitch;
} ulysses_a2a_desc_t;

/* Create a context on CUDA device `device` for elements of `elem_bytes` bytes
 * (1, 2, 4 or 8; bf16 = 2, fp32 = 4). On success *out holds a new context that
 * ulysses_a2a_destroy must release. Allocates a few bytes of device memory.
 * For testing, two environment variables set the context's initial knobs
 * (ulysses_a2a_set_path / ulysses_a2a_set_tuning override them later):
 * ULYSSES_A2A_FORCE_PATH = auto | tma | vec, and ULYSSES_A2A_CTAS_PER_SM =
 * 1..32 (the ctas_per_sm knob). A malformed value makes creation fail with
 * ULYSSES_A2A_ERR_INVALID. */
int ulysses_a2a_create(ulysses_a2a_ctx **out, int device, int elem_bytes);

/* Release a context. NULL is accepted. Always consumes the handle, even when a
 * CUDA cleanup call reports an error (returned as ULYSSES_A2A_ERR_CUDA); never
 * call it twice on the same pointer. Waits for the context's own work first. */
int ulysses_a2a_destroy(ulysses_a2a_ctx *ctx);

/* The re-layout (FastVideo API docs, ulysses_a2a `run_armed`: output shapes of
 * both modes, the mode-0-local argument tuple, and the chunked loop).
 *   in_slabs  : host array of w device pointers, the input slab of each rank.
 *   out_slabs : host array of w device pointers, caller-allocated outputs. No
 *               output may overlap any input or any other output.
 *   B, S_local, H, D : mode-0-local sizes, all >= 0, H % w == 0. If any is
 *               0 the re-layout is empty: the call returns ULYSSES_A2A_OK
 *               without launching anything (slab pointers may be NULL).
 *   w         : rank count, 1 <= w <= ULYSSES_A2A_MAX_W (w = 1 is a copy).
 *   mode      : 0 (scatter heads, gather sequence) or 1 (the inverse).
 *   chunked   : 0 = one launch over all B planes; 1 = the per-plane variant:
 *               one launch per plane b on the one-plane views, in stream
 *               order, so plane b is complete before plane b+1 starts;
 *               2 = the per-plane variant through a staging window: plane b
 *               of every input slab is first copied into a context-owned
 *               device window (grown on demand, reused plane after plane),
 *               then re-laid out from the window into plane b of the outputs
 *               (twice the memory traffic of 0 and 1). Same bytes in the
 *               outputs whichever is chosen.
 *   stream    : a cudaStream_t (NULL = legacy default stream).
 * With chunked = 0 or 1 the call is asynchronous on `stream`: it neither
 * synchronises the host nor allocates device memory. With chunked = 2, a call
 * whose planes need a larger window than the context holds first synchronises
 * `stream`, frees the old window and allocates a larger one (cudaMalloc), then
 * queues its work; calls whose planes fit the current window neither allocate
 * nor synchronise. */
int ulysses_a2a_run(ulysses_a2a_ctx *ctx, const void *const *in_slabs,
                    void *const *out_slabs, int64_t B, int64_t S_local,
                    int64_t H, int64_t D, int w, int mode, int chunked,
                    void *stream);

/* ulysses_a2a_run with the arguments in a descriptor (adds row_pitch). */
int ulysses_a2a_run_ex(ulysses_a2a_ctx *ctx, const ulysses_a2a_desc_t *desc,
                       void *stream);

/* Same operation on HOST slabs (pageable or pinned): copies every input to
 * context-owned device buffers, runs the re-layout on `stream`, copies every
 * output back, and returns once out_slabs hold the result. Device buffers grow
 * on demand and are kept until ulysses_a2a_destroy. */
int ulysses_a2a_run_host(ulysses_a2a_ctx *ctx, const void *const *in_slabs,
                         void *const *out_slabs, int64_t B, int64_t S_local,
                         int64_t H, int64_t D, int w, int mode, int chunked,
                         void *stream);

/* Human-readable reason for the last failed call on ctx ("" if none). The
 * string belongs to ctx and stays valid until the next call on it. */
const char *ulysses_a2a_last_error(const ulysses_a2a_ctx *ctx);

/* Synchronise `stream` and read (then clear) the context's device status word.
 * Returns ULYSSES_A2A_ERR_TIMEOUT if any kernel launched by this context gave
 * up a bounded wait since the last check, else ULYSSES_A2A_OK. */
int ulysses_a2a_status(ulysses_a2a_ctx *ctx, void *stream);

/* Failure-path self-test: launches on `stream` a one-thread kernel that waits
 * on an mbarrier nothing ever arrives on, through the same bounded wait the
 * copy kernel uses, but limited to limit_us microseconds (1..2 000 000); on
 * expiry it records the timeout in the context's status words exactly as the
 * copy kernel would. The next ulysses_a2a_status then returns
 * ULYSSES_A2A_ERR_TIMEOUT, and the context stays usable. Nothing but the
 * status words is touched. */
int ulysses_a2a_selftest_wait_timeout(ulysses_a2a_ctx *ctx, uint32_t limit_us,
                                      void *stream);

/* Force a copy path (ULYSSES_A2A_PATH_*) for later runs; AUTO restores the
 * default choice. A forced path that cannot express a shape makes run fail
 * with ULYSSES_A2A_ERR_UNSUPPORTED instead of silently switching. */
int ulysses_a2a_set_path(ulysses_a2a_ctx *ctx, int path);

/* Speed knobs. Results never depend on them, only speed does; every field
 * left at its "default" value keeps the library's choice. */
typedef struct ulysses_a2a_tuning_t {
    int32_t rows_per_tile;  /* S_tile cap, 1..256; 0 = default                */
    int32_t ctas_per_sm;    /* CTAs per SM, 1..32; 0 = default. TMA
                               chunk schedule: a cap on resident CTAs per
                               SM, enforced by reserving shared memory
                               (default: about 100 KB of tiles in flight
                               per SM); persistent TMA grid: its size;
                               VEC: a grid-stride grid of this many per SM
                               (default: one CTA per unit)                */
    int32_t stages;         /* TMA: shared-memory tiles per CTA, 1..32, split
                               evenly over the producers; 0 = default      */
    int32_t lookahead;      /* TMA: loads in flight per producer; 0 = default */
    int32_t producers;      /* TMA: producer warps per CTA, 1..8; 0 = default */
    int32_t order;          /* unit numbering: 0 = destination rank r
                               outermost, 1 = innermost; -1 = default      */
    int32_t chunk_units;    /* TMA schedule: 0 = persistent grid (static
                               round robin); n > 0 = n consecutive units per
                               CTA; -1 = default (one unit per producer;
                               one producer by default)                   */
    int32_t host_chunks;    /* host-buffer entry point: sequence chunks its
                               copies and kernels are pipelined over, 1..64;
                               0 = default                                */
    int32_t staged_form;    /* STAGED path: 0 = the fixed-phase form where it
                               applies (default; see plan_t.fixed_phase),
                               1 = the per-piece form always              */
} ulysses_a2a_tuning_t;

/* Apply tuning to later runs (NULL restores every default). Values outside
 * the ranges above are rejected with ULYSSES_A2A_ERR_INVALID. */
int ulysses_a2a_set_tuning(ulysses_a2a_ctx *ctx, const ulysses_a2a_tuning_t *tuning);

/* The context's current forced path (ULYSSES_A2A_PATH_*) and tuning, as set
 * by the environment at creation, ulysses_a2a_set_path and
 * ulysses_a2a_set_tuning (default fields keep their "default" values). Either
 * output may be NULL. */
int ulysses_a2a_get_settings(const ulysses_a2a_ctx *ctx, int32_t *path,
                             ulysses_a2a_tuning_t *tuning);

/* Kernel launches this context has issued since creation. */
uint64_t ulysses_a2a_launch_count(const ulysses_a2a_ctx *ctx);

/* Host-only planning: validates the arguments exactly as ulysses_a2a_run does
 * (except the device-residency check, which needs a GPU) and reports the path
 * and geometry it would use. Makes no CUDA call, so it runs without a GPU.
 * Pointer values are only compared and tested for alignment, never read.
 * forced_path as in ulysses_a2a_set_path; tuning as in ulysses_a2a_set_tuning
 * (NULL = defaults); num_sms = streaming multiprocessors of the target device
 * (148 on B200). On failure writes a message of at most errlen bytes into err
 * (if non-NULL). */
int ulysses_a2a_plan(const void *const *in_slabs, void *const *out_slabs,
                     int64_t B, int64_t S_local, int64_t H, int64_t D, int w,
                     int mode, int chunked, int elem_bytes, int forced_path,
                     const ulysses_a2a_tuning_t *tuning, int num_sms,
                     ulysses_a2a_plan_t *out, char *err, size_t errlen);

/* Allocation-free variant of ulysses_a2a_run (the pages have no counterpart:
 * this entry point exists for this library's users, not for the method).
 *
 * Who needs it: callers that must not allocate device memory themselves, e.g.
 * a process whose device memory is owned by another allocator under a fixed
 * budget, or host code running where a cudaMalloc/cudaFree (which may
 * synchronise the whole device) is not allowed. ulysses_a2a_create allocates
 * the TMA kernel's status records; this call needs no context and allocates
 * nothing: it keeps those records in a file-scope static device array of 64
 * records x 16 bytes (1 KiB), one record per TMA kernel launch, which every
 * GPU that loads the library holds until the process exits. (The vector-path
 * kernel has no bounded wait and uses no record.)
 *
 * Arguments and layout as ulysses_a2a_run, plus elem_bytes (1, 2, 4 or 8). It
 * runs on the CURRENT CUDA device, which must hold every slab. The caller still
 * owns all inputs and outputs.
 *   wait = 0 : return once the work is queued on `stream`. Nothing reads
 *              the status records of such a call, so a bounded wait that
 *              gave up in it is never reported (the next call clears them).
 *   wait = 1 : also synchronise `stream` and check the status records;
 *              returns ULYSSES_A2A_ERR_TIMEOUT if a kernel gave up a wait.
 *   err      : optional buffer (errlen bytes) for a message on failure.
 * Limit: a chunked call on the TMA path launches once per plane and needs one
 * record per plane, so such calls over more than 64 planes are rejected with
 * ULYSSES_A2A_ERR_UNSUPPORTED and a message (unchunked calls need one record,
 * vector-path calls none).
 *
 * The first call on a device also does a one-time set-up for that device
 * (resolving the array's device address and the kernels' shared-memory limit);
 * make that first call before any stream capture. A set-up that fails is not
 * remembered: the next call on that device tries it again. Every call shares
 * the array and the array keeps the last call's contents: each call clears the
 * records it uses, on `stream`, before its kernels run, so calls whose work
 * overlaps on the GPU (other streams, other host threads) race on the records. */
int ulysses_a2a_run_noalloc(const void *const *in_slabs, void *const *out_slabs,
                            int64_t B, int64_t S_local, int64_t H, int64_t D,
                            int w, int mode, int chunked, int elem_bytes,
                            void *stream, int wait, char *err, size_t errlen);

/* ulysses_a2a_plan for a descriptor (adds row_pitch). */
int ulysses_a2a_plan_ex(const ulysses_a2a_desc_t *desc, int elem_bytes,
                        int forced_path, const ulysses_a2a_tuning_t *tuning,
                        int num_sms, ulysses_a2a_plan_t *out, char *err,
                        size_t errlen);

/* ---- multi-GPU exchange through published windows ----------------------
 *
 * One process per GPU, w ranks. Each rank owns a device window that every
 * other rank maps (CUDA IPC, or directly when the ranks share a process), in
 * the manner of the FastVideo API docs' ulysses_a2a communicator: a window
 * built once and reused call after call and plane after plane (`run_armed`,
 * chunked branch), rebuilt when a call needs more bytes (`try_all_to_all_4D`,
 * window grow), and torn down collectively (`close`). The pypto-lib pull
 * request "pipeline HCA AllToAll into O-A" publishes each rank's output into a
 * distributed window and has consumers load from it after a handshake; the
 * exchange here follows the same order:
 *
 *   1. ulysses_a2a_peer_publish: copy this rank's input slab (or one plane of
 *      it) into this rank's window, dense;
 *   2. a barrier: every rank's publish is complete;
 *   3. ulysses_a2a_peer_pull: one kernel reads this rank's share out of every
 *      rank's window (peer loads over NVLink) and writes this rank's output
 *      slab, with the same element map as ulysses_a2a_run, of which it is the
 *      launch restricted to output slab `rank`;
 *   4. a barrier: every rank's pull is complete, so the windows may be
 *      published into again.
 *
 * The barriers are the caller's (a stream-ordered collective such as a
 * one-element NCCL all-reduce on the same stream, or a stream synchronise plus
 * a host barrier): this library launches no kernel that waits for another GPU.
 * Chunked calls pass one-plane views (B = 1) and repeat 1-4 per plane.
 * Sizes are mode-0-local as everywhere in this header; in mode 0 rank k's
 * input is x_k [B, S_local, H, D] (row pitch allowed) and its output out_k
 * [B, S_local*w, H/w, D]; in mode 1 the input is [B, S_local*w, H/w, D] and
 * the output [B, S_local, H, D] (row pitch allowed). A window must hold one
 * input slab of the largest call: B*S_local*H*D*elem_bytes bytes. The output
 * never aliases a window.
 */
typedef struct ulysses_a2a_peer ulysses_a2a_peer; /* opaque */

#define ULYSSES_A2A_PEER_HANDLE_BYTES 128 /* size of one exchanged record */

/* Allocate this rank's window (window_bytes >= 1, on ctx's device) and write
 * its exchange record, ULYSSES_A2A_PEER_HANDLE_BYTES bytes, into handle_out.
 * The caller gathers every rank's record, in rank order, to every rank (for
 * example with an all-gather) and passes them to ulysses_a2a_peer_open. The
 * peer object uses ctx (element size, device, status) and must be destroyed
 * before it. 1 <= world <= ULYSSES_A2A_MAX_W, 0 <= rank < world. */
int ulysses_a2a_peer_create(ulysses_a2a_ctx *ctx, int rank, int world,
                            size_t window_bytes, ulysses_a2a_peer **out,
                            void *handle_out);

/* Map every other rank's window. handles: world records in rank order, as
 * written by each rank's ulysses_a2a_peer_create. Records must agree on
 * world, element size and window size, and record k must come from rank k;
 * a record from this same process is used directly (its device gets peer
 * access if it differs from ctx's), any other is opened with CUDA IPC.
 * Fails without mapping anything if a record is malformed. */
int ulysses_a2a_peer_open(ulysses_a2a_peer *peer, const void *handles);

/* Step 1: copy this rank's input slab into its own window, from byte
 * window_offset on (asynchronous on stream). mode 0: in_local is
 * [B, S_local, H, D] with row_pitch (0 = dense, else >= H*D elements between
 * rows, as in ulysses_a2a_desc_t); mode 1: in_local is [B, S_local*w, H/w, D]
 * dense and row_pitch must be 0. The window receives the dense slab.
 * window_offset is a multiple of the element size, and the slab must fit in
 * the window after it. Several slabs can share a window at different offsets
 * (for example the T tensors of a head-packed exchange).
 * If in_local is the window itself at that offset holding the dense slab, the
 * slab was written in place and nothing is copied or launched (zero-copy
 * publish: the producer of the slab writes into the window directly, after
 * the barrier of step 4 of the previous exchange). */
int ulysses_a2a_peer_publish(ulysses_a2a_peer *peer, const void *in_local,
                             int64_t B, int64_t S_local, int64_t H, int64_t D,
                             int mode, int64_t row_pitch, size_t window_offset,
                             void *stream);

/* Step 3: write this rank's output slab from every rank's published window,
 * each read from byte window_offset on (asynchronous on stream; VEC kernel,
 * peer loads). out_local is on ctx's device, caller-owned, and overlaps no
 * window. row_pitch belongs to the [B, S_local, H, D] side: in mode 0 that is
 * the windows (read with that pitch: e.g. tensor t of a head-packed slab
 * published whole, with row_pitch = T*H*D and window_offset = t*H*D*elem_bytes)
 * and out_local is [B, S_local*w, H/w, D] dense; in mode 1 it is out_local,
 * [B, S_local, H, D] with row_pitch (0 = dense), and the windows hold dense
 * [B, S_local*w, H/w, D] slabs. Requires ulysses_a2a_peer_open to have
 * succeeded. */
int ulysses_a2a_peer_pull(ulysses_a2a_peer *peer, void *out_local, int64_t B,
                          int64_t S_local, int64_t H, int64_t D, int mode,
                          int64_t row_pitch, size_t window_offset, void *stream);

/* Step 3 for T tensors packed along the head dimension (for example q, k and
 * v of a packed projection output), in ONE kernel launch for all T (the
 * launch of ulysses_a2a_run_ex with ntensors = T, restricted to this rank's
 * outputs). 1 <= ntensors, ntensors * world <= ULYSSES_A2A_MAX_W.
 *   mode 0: every window holds its rank's packed [B, S_local, T, H, D] slab,
 *           dense, from byte window_offset on (published with T*H heads);
 *           out_local holds T device pointers, out_local[t] receiving this
 *           rank's dense [B, S_local*w, H/w, D] slab of tensor t.
 *   mode 1: every window holds T dense [B, S_local*w, H/w, D] slabs, tensor
 *           t's at byte window_offset + t*B*S_local*H*D*elem_bytes;
 *           out_local[0] receives this rank's dense packed [B, S_local, T, H,
 *           D] slab.
 * Same bytes as T calls of ulysses_a2a_peer_pull with row pitch T*H*D and
 * the matching window offsets. Asynchronous on stream; VEC kernel, peer
 * loads; no output overlaps a window. */
int ulysses_a2a_peer_pull_packed(ulysses_a2a_peer *peer, void *const *out_local,
                                 int ntensors, int64_t B, int64_t S_local,
                                 int64_t H, int64_t D, int mode,
                                 size_t window_offset, void *stream);

/* Base address of rank k's window as this process sees it (NULL if k is out
 * of range or not mapped yet), and the window size in bytes. */
void *ulysses_a2a_peer_window(const ulysses_a2a_peer *peer, int rank);
size_t ulysses_a2a_peer_window_bytes(const ulysses_a2a_peer *peer);

/* Unmap the other ranks' windows (synchronising ctx's device first); the own
 * window stays. Call it on every rank, then barrier, then destroy: a window
 * must not be freed while a peer still maps it. Idempotent. */
int ulysses_a2a_peer_close(ulysses_a2a_peer *peer);

/* Close (if not done) and free the own window; consumes the handle even when
 * a CUDA call reports an error. NULL is accepted. */
int ulysses_a2a_peer_destroy(ulysses_a2a_peer *peer);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* ULYSSES_A2A_H */
