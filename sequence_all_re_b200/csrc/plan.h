// plan.h - host-only argument checks and work geometry for the Ulysses 4D
// all-to-all re-layout (FastVideo API docs, device_communicators/ulysses_a2a,
// `run_armed`: shapes of both modes and the per-plane chunked loop).
//
// Nothing here touches CUDA: the same code validates ulysses_a2a_run's
// arguments and answers ulysses_a2a_plan on a machine without a GPU.
//
// Work decomposition. For ranks r (destination head group) and j (source
// sequence shard), plane b and sequence tile t, one work unit moves rows
// s in [t*S_tile, min((t+1)*S_tile, S_local)) of the (r, b, j) block:
//   strided side  [B, S_local, H, D]     : rows of L = (H/w)*D elements,
//                                          stride H*D, at head offset r*L;
//   gathered side [B, S_local*w, H/w, D] : the same rows, contiguous, at
//                                          sequence offset j*S_local.
// Mode 0 reads the strided side and writes the gathered side; mode 1 the
// reverse. Units are numbered (r, b, j, t) with t fastest, so consecutive
// CTAs touch consecutive bytes of the contiguous side.
#pragma once

#include <cstdint>
#include <cstdio>
#include <string>

#include "ulysses_a2a.h"

namespace ua2a {

// Bytes of one work unit the planner aims for: a shared-memory stage of the
// TMA path, a CTA's unit of the VEC path (measured on B200: 12 KB units, one
// per short-lived CTA, beat 8 KB and below by 3-35 % and 16-64 KB by 1-7 %).
constexpr int64_t kTmaTileTargetBytes = 8 * 1024;
constexpr int64_t kTileTargetBytes = 12 * 1024;
// Largest TMA tile; a single row longer than this goes to the VEC path.
constexpr int64_t kTmaMaxTileBytes = 64 * 1024;
// Dynamic shared memory the TMA ring may use per CTA by default (of 227 KB).
constexpr int64_t kTmaSmemBudget = 192 * 1024;
constexpr int64_t kTmaSmemMax = 220 * 1024;
// B200 (sm_100): shared memory an SM can give its resident CTAs, and the part
// of it the driver reserves per CTA.
constexpr int64_t kSmemPerSm = 228 * 1024;
constexpr int64_t kSmemReservedPerCta = 1024;
// Chunk schedule default: one producer warp and one unit per CTA, with the
// CTAs resident on an SM capped so that about this many tile bytes are in
// flight per SM (measured on B200: ~90-110 KB beats both the uncapped ~190 KB
// and 60-80 KB by 1-15 %).
constexpr int64_t kTmaInflightPerSm = 100 * 1024;
constexpr int kTmaMaxStages = 32;            // all producers together
constexpr int kTmaMaxProducers = 8;          // producer warps per CTA
constexpr int kTmaDefaultProducers = 4;
constexpr int kTmaStagesPerProducer = 4;     // default sub-ring depth
constexpr int kTmaDefaultCtasPerSm = 1;
constexpr int kTmaMaxBoxDim = 256;
constexpr int kVecBlock = 256;
// CTAs of the VEC kernel resident per SM (its launch bound). By default the
// VEC grid has one CTA per unit, and the hardware hands CTAs to SMs as they
// free up, so no SM is left with a tail of units.
constexpr int kVecResidentCtasPerSm = 6;
// Re-aligning (staged) path: strided-side bytes per work unit, the shared
// memory one CTA may use, and its threads.
constexpr int64_t kStageTileTargetBytes = 16 * 1024;
constexpr int64_t kStageSmemMax = 96 * 1024;
constexpr int kStageBlock = 256;
// Its fixed-phase form (kernels_phase.cuh): strided-side bytes per work unit,
// and the fewest of the kStageBlock threads that must move strided chunks (a
// multiple of HDE / gcd(HDE, 16) of them do). Measured on B200 with this
// constant rebuilt at each size (6- and 12-byte runs, mode 0 / mode 1 of the
// copy bandwidth, regions an odd number of chunks apart): units of 8 KB
// 0.52 / 0.43 and 0.68 / 0.67, 16 KB 0.72 / 0.53 and 0.87 / 0.83, 32 KB
// 0.74 / 0.62 and 0.91 / 0.89, 48 KB 0.70 / 0.65 and 0.76 / 0.79.
constexpr int64_t kPhaseTileTargetBytes = 32 * 1024;
// With 128 or more movers the fixed-phase form still beats the per-piece one
// (measured, mode 0 / mode 1: 135 movers, 10-byte runs 0.52 / 0.59 against
// 0.43 / 0.37; 175 movers, 5-byte runs 0.44 / 0.41 against 0.23 / 0.21); a
// phase period of at most 256 chunks always leaves more than 128.
constexpr int kPhaseMinMovers = 128;
// AUTO moves launches of at most this many payload bytes with the vector
// kernel even where TMA could take them: measured on B200 in CUDA-graph
// replays, a vector launch costs about 0.6-1 us less (128 KiB: 1.3-1.5 us
// against 2.0 us; 8 MiB: 2.9 against 3.7 us; 64 MiB: 19.5 against 20.9 us)
// since its CTAs retire once their stores are issued, while a TMA tile waits
// for its load and then for its store to read shared memory; from 192 MiB on
// the two paths are within 2 % of each other.
constexpr int64_t kVecSmallLaunchBytes = int64_t(64) << 20;
// Smallest vector unit: small launches get units of payload / (2 * SMs),
// down to this size, so that every SM has work.
constexpr int64_t kVecMinTileBytes = 2 * 1024;
// AUTO re-aligns through shared memory what the vector kernel would move in
// pieces of at most kStageMaxPiece bytes, and 8-byte-granular runs when the
// fixed-phase form applies. Measured on B200 (mode 0 / mode 1 of the copy
// bandwidth, bench.py --staged-forms): 4-, 2- and 1-byte vectors reach
// 0.16-0.53 against 0.44-0.98 for the fixed-phase form; 8-byte vectors 0.44 /
// 0.45 on 8-byte runs, 0.77 / 0.81 on 24, 0.85 / 0.58 on 40, 0.89 / 0.71 on
// 72, 0.90 / 0.84 on 104, 0.91 / 0.92 on 136 and 0.91 / 0.94 on 200, against
// 0.99-1.03 / 0.96-1.03 for the fixed-phase form (its mode-0 gather).
constexpr int kStageMaxPiece = 4;
// Unit numbering: 0 = destination rank outermost, 1 = innermost.
constexpr int kDefaultOrder = 1;
// Host-buffer entry point: sequence chunks its H2D copies, kernels and D2H
// copies are pipelined over (payloads below kHostChunkMinBytes use one).
constexpr int kHostMaxChunks = 64;
constexpr int kHostDefaultChunks = 8;
constexpr int64_t kHostChunkMinBytes = 8 << 20;
// TMA schedule: by default a grid of ceil(units / n) short-lived CTAs, each
// taking n consecutive units, one per producer warp, with a one-tile ring per
// producer (default: one producer, n = 1). The hardware hands CTAs to SMs as
// they finish, so there is no static tail imbalance, and the residency cap
// (kTmaInflightPerSm) sets how many share an SM. chunk_units = 0 selects a
// persistent grid (static round robin) with deeper rings instead.

struct Tuning {
  int rows_per_tile = 0;  // 0 = default
  int ctas_per_sm = 0;
  int stages = 0;
  int lookahead = 0;      // TMA loads in flight per producer (0 = default: S - S/2)
  int producers = 0;      // TMA producer warps per CTA (0 = default)
  int order = -1;         // unit numbering (-1 = default)
  int chunk_units = -1;   // TMA: units per CTA (0 = persistent grid, -1 = default)
  int host_chunks = 0;    // host-buffer path pipeline depth (0 = default)
  int staged_form = 0;    // staged path: 0 = fixed-phase form where it applies, 1 = per-piece
};

inline bool mul_overflows(int64_t a, int64_t b, int64_t* out) {
  return __builtin_mul_overflow(a, b, out);
}

inline void set_err(std::string* err, const char* fmt, long long a = 0, long long b = 0) {
  if (!err) return;
  char buf[256];
  std::snprintf(buf, sizeof(buf), fmt, a, b);
  *err = buf;
}

// [lo, hi) ranges intersect?
inline bool overlaps(uintptr_t a, uintptr_t a_end, uintptr_t b, uintptr_t b_end) {
  return a < b_end && b < a_end;
}

// Why the TMA path cannot take a shape (nullptr if it can).
inline const char* tma_blocker(const void* const* in, void* const* out, int64_t B,
                               int64_t S, int64_t H, int64_t D, int w, int E,
                               int64_t row_bytes, int64_t pitch) {
  const int64_t Hw = H / w;
  if ((pitch * E) % 16 != 0) return "the row pitch is not a multiple of 16 bytes";
  if (w > ULYSSES_A2A_MAX_W_TMA) return "w exceeds the TMA path's rank limit";
  if (D > kTmaMaxBoxDim || Hw > kTmaMaxBoxDim) return "D or H/w exceeds a TMA box dimension (256)";
  if ((D * E) % 16 != 0) return "D*elem_bytes is not a multiple of 16 bytes";
  if (row_bytes > kTmaMaxTileBytes) return "one row run exceeds the TMA tile limit";
  if (S > INT32_MAX || B > INT32_MAX) return "S_local or B exceeds a TMA coordinate";
  // global strides must stay below 2^40 bytes: the largest is one plane
  if (S * pitch * E >= (int64_t(1) << 40)) return "plane stride exceeds the TMA stride limit";
  for (int k = 0; k < w; ++k) {
    if ((reinterpret_cast<uintptr_t>(in[k]) & 15u) != 0 ||
        (reinterpret_cast<uintptr_t>(out[k]) & 15u) != 0)
      return "a slab base address is not 16-byte aligned";
  }
  return nullptr;
}

// Peeled vector path: runs of at least this many bytes (shorter ones are
// mostly head and tail).
constexpr int64_t kPeelMinRunBytes = 64;

// Offsets past a 16-byte boundary shared by every input slab (*a_in) and by
// every output slab (*a_out) of a call whose runs (run_bytes) and rows
// (pitch_bytes) are whole multiples of 16 bytes: every run then starts *a_in
// bytes past a boundary on the input side and *a_out on the output side.
// False when the slabs of a side differ, or a run or a row is no multiple of 16.
inline bool side_offsets(const void* const* in, int nin, void* const* out, int nout,
                         int64_t run_bytes, int64_t pitch_bytes, int* a_in, int* a_out) {
  if (run_bytes % 16 != 0 || pitch_bytes % 16 != 0 || nin < 1 || nout < 1) return false;
  const uintptr_t ai = reinterpret_cast<uintptr_t>(in[0]) & 15u;
  const uintptr_t ao = reinterpret_cast<uintptr_t>(out[0]) & 15u;
  for (int k = 0; k < nin; ++k)
    if ((reinterpret_cast<uintptr_t>(in[k]) & 15u) != ai) return false;
  for (int k = 0; k < nout; ++k)
    if ((reinterpret_cast<uintptr_t>(out[k]) & 15u) != ao) return false;
  *a_in = (int)ai;
  *a_out = (int)ao;
  return true;
}

// Geometry of the re-aligning (staged) path for runs of R bytes, ng head
// groups per strided row (HDE = ng * R bytes) and S_local rows: the rows per
// unit (about kStageTileTargetBytes of strided-side bytes, kPhaseTileTargetBytes
// in the fixed-phase form, or rows_cap when set), the 16-byte chunks scanned
// per strided row (Cs) and per gathered range (Cg), and the shared memory of a
// CTA: ng regions of RS bytes and ng 4-byte region offsets. RS is 16*Cg
// rounded up to an odd number of 16-byte chunks, so that consecutive regions
// start in different shared-memory banks; in the fixed-phase form with at most
// 4 regions, to a multiple of 128 bytes instead: one warp's 32 strided chunks
// then cover at least 128 bytes of every region, and regions that start in
// the same bank gave the fewest conflicts (modelled: 1.5 against 3.0
// wavefronts per access on 6-byte runs; measured: 0.81 / 0.64 against
// 0.74 / 0.62 of the copy bandwidth).
// Returns false if not even one row fits kStageSmemMax.
struct StageGeometry {
  int64_t rows = 0, tiles = 0, Cs = 0, Cg = 0, RS = 0, smem_bytes = 0;
};

inline bool stage_geometry(int64_t R, int64_t ng, int64_t S, int rows_cap, StageGeometry* g,
                           bool fixed_phase = false, bool image = false) {
  const int64_t HDE = ng * R;
  if (R < 1 || ng < 1 || S < 1 || HDE >= (int64_t(1) << 30)) return false;
  int64_t rows = rows_cap > 0 ? rows_cap
                              : (fixed_phase ? kPhaseTileTargetBytes : kStageTileTargetBytes) / HDE;
  if (rows < 1) rows = 1;
  if (rows > S) rows = S;
  for (; rows >= 1; rows = rows > 1 ? rows / 2 : 0) {
    const int64_t Cg = (rows * R + 30) / 16;
    const int64_t RS = 16 * (fixed_phase && ng <= 4 ? (Cg + 7) / 8 * 8 : (Cg % 2 ? Cg : Cg + 1));
    // the fixed-phase form's mode-0 gather (pieces of 4 bytes or more) holds
    // the strided segment's 16-byte chunks as loaded (at most
    // (rows * HDE + 30) / 16 of them, swizzled within 128-byte blocks); every
    // other launch holds the ng regions
    const int64_t smem = image ? (16 * ((rows * HDE + 30) / 16) + 127) / 128 * 128 : ng * RS + 4 * ng;
    if (smem <= kStageSmemMax && rows * HDE < (int64_t(1) << 30)) {
      g->rows = rows;
      g->tiles = (S + rows - 1) / rows;
      g->Cs = (HDE + 30) / 16;
      g->Cg = Cg;
      g->RS = RS;
      g->smem_bytes = (smem + 15) / 16 * 16;
      return true;
    }
  }
  return false;
}

// Threads of a kStageBlock-thread CTA that move strided chunks in the
// fixed-phase form for strided rows of HDE bytes: the largest multiple of
// HDE / gcd(HDE, 16) up to kStageBlock (0 when there is none).
inline int64_t phase_movers(int64_t HDE) {
  int64_t g = 16;
  while (HDE % g != 0) g >>= 1;
  const int64_t period = HDE / g;
  return period <= kStageBlock ? period * (kStageBlock / period) : 0;
}

// Public tuning struct -> internal knobs, with range checks (NULL = defaults).
inline bool tuning_from(const ulysses_a2a_tuning_t* t, Tuning* out, std::string* err) {
  *out = Tuning{};
  if (t == nullptr) return true;
  auto bad = [&](const char* what) {
    if (err) *err = std::string("tuning value out of range: ") + what;
    return false;
  };
  if (t->rows_per_tile < 0 || t->rows_per_tile > kTmaMaxBoxDim) return bad("rows_per_tile");
  if (t->ctas_per_sm < 0 || t->ctas_per_sm > 32) return bad("ctas_per_sm");
  if (t->stages < 0 || t->stages > kTmaMaxStages) return bad("stages");
  if (t->lookahead < 0 || t->lookahead > kTmaMaxStages) return bad("lookahead");
  if (t->producers < 0 || t->producers > kTmaMaxProducers) return bad("producers");
  if (t->order < -1 || t->order > 1) return bad("order");
  if (t->chunk_units < -1) return bad("chunk_units");
  if (t->host_chunks < 0 || t->host_chunks > kHostMaxChunks) return bad("host_chunks");
  if (t->staged_form < 0 || t->staged_form > 1) return bad("staged_form");
  out->rows_per_tile = t->rows_per_tile;
  out->ctas_per_sm = t->ctas_per_sm;
  out->stages = t->stages;
  out->lookahead = t->lookahead;
  out->producers = t->producers;
  out->order = t->order;
  out->chunk_units = t->chunk_units;
  out->host_chunks = t->host_chunks;
  out->staged_form = t->staged_form;
  return true;
}

// Validate and plan one call. Returns a ULYSSES_A2A_* status.
// row_pitch: elements between consecutive (b, s) rows of the [B, S, H, D]
// side (0 = dense, H*D); that side's planes are S*row_pitch elements apart.
// only_out >= 0: the call writes the output slab(s) of rank only_out alone
// (VEC path): slab only_out, or with ntensors = T > 1 in mode 0 the T slabs
// t*w + only_out; the other out[] entries are neither checked nor used, and
// units counts those slabs' blocks only.
// ntensors = T > 1: T tensors packed along the head dimension of the
// [B, S, H, D] side ([B, S, T, H, D], rows of T*H*D elements), re-laid out in
// one launch (VEC path). That side then has w slabs and the other T*w, tensor-
// major: slab t*w + r is tensor t's [B, S*w, H/w, D] slab of rank r.
inline int make_plan(const void* const* in, void* const* out, int64_t B, int64_t S,
                     int64_t H, int64_t D, int w, int mode, int chunked, int E,
                     int forced_path, const Tuning& tune, int num_sms,
                     ulysses_a2a_plan_t* p, std::string* err, int64_t row_pitch = 0,
                     int only_out = -1, int ntensors = 1) {
  if (p == nullptr) { set_err(err, "plan output is NULL"); return ULYSSES_A2A_ERR_INVALID; }
  *p = ulysses_a2a_plan_t{};
  if (in == nullptr || out == nullptr) {
    set_err(err, "in_slabs/out_slabs array is NULL");
    return ULYSSES_A2A_ERR_INVALID;
  }
  if (w < 1 || w > ULYSSES_A2A_MAX_W) {
    set_err(err, "w=%lld outside [1, %lld]", w, ULYSSES_A2A_MAX_W);
    return ULYSSES_A2A_ERR_INVALID;
  }
  if (!(E == 1 || E == 2 || E == 4 || E == 8)) {
    set_err(err, "elem_bytes=%lld not in {1,2,4,8}", E);
    return ULYSSES_A2A_ERR_INVALID;
  }
  if (mode != 0 && mode != 1) { set_err(err, "mode=%lld not 0 or 1", mode); return ULYSSES_A2A_ERR_INVALID; }
  if (only_out >= w || (only_out >= 0 && forced_path != ULYSSES_A2A_PATH_VEC)) {
    set_err(err, "one-output plan: slab %lld of %lld, VEC path required", only_out, w);
    return ULYSSES_A2A_ERR_INVALID;
  }
  if (ntensors < 1 || (int64_t)ntensors * w > ULYSSES_A2A_MAX_W) {
    set_err(err, "ntensors=%lld: need 1 <= ntensors and ntensors*w <= %lld", ntensors,
            ULYSSES_A2A_MAX_W);
    return ULYSSES_A2A_ERR_INVALID;
  }
  if (ntensors > 1 && chunked == 2) {
    set_err(err, "packed tensors are not staged through the window (chunked must be 0 or 1)");
    return ULYSSES_A2A_ERR_UNSUPPORTED;
  }
  if (chunked < 0 || chunked > 2) { set_err(err, "chunked=%lld not 0, 1 or 2", chunked); return ULYSSES_A2A_ERR_INVALID; }
  if (B < 0 || S < 0 || H < 0 || D < 0) {
    set_err(err, "sizes must be >= 0 (B, S_local, H, D)");
    return ULYSSES_A2A_ERR_INVALID;
  }
  if (H % w != 0) { set_err(err, "H=%lld not divisible by w=%lld", H, w); return ULYSSES_A2A_ERR_INVALID; }
  if (B == 0 || S == 0 || H == 0 || D == 0) {
    // an empty re-layout: nothing to read or write, nothing to launch (slab
    // pointers may be NULL)
    if (forced_path < ULYSSES_A2A_PATH_AUTO || forced_path > ULYSSES_A2A_PATH_STAGED) {
      set_err(err, "unknown path %lld", forced_path);
      return ULYSSES_A2A_ERR_INVALID;
    }
    p->path = forced_path == ULYSSES_A2A_PATH_AUTO ? ULYSSES_A2A_PATH_VEC : forced_path;
    p->row_pitch = row_pitch > 0 ? row_pitch : (int64_t)ntensors * H * D;
    return ULYSSES_A2A_OK;
  }
  if (forced_path < ULYSSES_A2A_PATH_AUTO || forced_path > ULYSSES_A2A_PATH_STAGED) {
    set_err(err, "unknown path %lld", forced_path);
    return ULYSSES_A2A_ERR_INVALID;
  }
  if (num_sms < 1) { set_err(err, "num_sms must be >= 1"); return ULYSSES_A2A_ERR_INVALID; }

  // sizes, overflow-checked
  int64_t plane_elems, slab_elems, slab_bytes, payload, tmp, HD, HDp;
  if (mul_overflows(S, H, &tmp) || mul_overflows(tmp, D, &plane_elems) ||
      mul_overflows(plane_elems, B, &slab_elems) || mul_overflows(slab_elems, E, &slab_bytes) ||
      mul_overflows(slab_bytes, (int64_t)w * ntensors, &payload) || payload > (int64_t(1) << 56) ||
      mul_overflows(H, D, &HD) || mul_overflows(HD, (int64_t)ntensors, &HDp)) {
    set_err(err, "slab sizes overflow");
    return ULYSSES_A2A_ERR_INVALID;
  }
  // HDp: elements of one (b, s) row of the [B, S, (T,) H, D] side
  const int64_t pitch = row_pitch == 0 ? HDp : row_pitch;
  if (pitch < HDp) {
    set_err(err, "row pitch %lld is smaller than a row (%lld elements)", pitch, HDp);
    return ULYSSES_A2A_ERR_INVALID;
  }
  // bytes spanned by one slab of the [B, S, H, D] side (gaps included)
  int64_t strided_bytes;
  if (mul_overflows(B * S - 1, pitch, &tmp) || mul_overflows(tmp + HDp, (int64_t)E, &strided_bytes) ||
      strided_bytes > (int64_t(1) << 56)) {
    set_err(err, "pitched slab extent overflows");
    return ULYSSES_A2A_ERR_INVALID;
  }
  const int64_t in_bytes = mode == 0 ? strided_bytes : slab_bytes;
  const int64_t out_bytes = mode == 0 ? slab_bytes : strided_bytes;
  // slab counts: w on the [B, S, (T,) H, D] side, T*w on the gathered side
  const int nin = mode == 0 ? w : w * ntensors;
  const int nout = mode == 0 ? w * ntensors : w;
  // outputs this call writes: all, or rank only_out's (one per tensor in mode 0)
  auto used_out = [&](int k) {
    return only_out < 0 || (mode == 0 ? k % w == only_out : k == only_out);
  };
  for (int k = 0; k < nin; ++k) {
    if (in[k] == nullptr) {
      set_err(err, "input slab pointer %lld is NULL", k);
      return ULYSSES_A2A_ERR_INVALID;
    }
  }
  for (int k = 0; k < nout; ++k) {
    if (used_out(k) && out[k] == nullptr) {
      set_err(err, "output slab pointer %lld is NULL", k);
      return ULYSSES_A2A_ERR_INVALID;
    }
  }
  // No output may overlap an input or another output (inputs may alias each
  // other). A pitched slab counts with its whole extent, gaps included.
  for (int k = 0; k < nout; ++k) {
    if (!used_out(k)) continue;
    const uintptr_t o = reinterpret_cast<uintptr_t>(out[k]);
    const uintptr_t oe = o + (uintptr_t)out_bytes;
    if (oe < o) { set_err(err, "output slab %lld wraps the address space", k); return ULYSSES_A2A_ERR_INVALID; }
    for (int m = 0; m < nin; ++m) {
      const uintptr_t i = reinterpret_cast<uintptr_t>(in[m]);
      if (overlaps(o, oe, i, i + (uintptr_t)in_bytes)) {
        set_err(err, "output slab %lld overlaps input slab %lld", k, m);
        return ULYSSES_A2A_ERR_OVERLAP;
      }
    }
    for (int m = 0; m < nout; ++m) {
      if (m != k && used_out(m)) {
        const uintptr_t q = reinterpret_cast<uintptr_t>(out[m]);
        if (overlaps(o, oe, q, q + (uintptr_t)out_bytes)) {
          set_err(err, "output slab %lld overlaps output slab %lld", k, m);
          return ULYSSES_A2A_ERR_OVERLAP;
        }
      }
    }
  }

  const int64_t Hw = H / w;
  const int64_t row_bytes = Hw * D * E;  // one contiguous run, L*E
  const char* blocker = only_out >= 0   ? "one-output launches use the VEC path"
                        : ntensors > 1 ? "packed launches use the VEC path"
                                       : tma_blocker(in, out, B, S, H, D, w, E, row_bytes, pitch);
  int path;
  if (forced_path == ULYSSES_A2A_PATH_TMA) {
    if (blocker) {
      if (err) *err = std::string("TMA path forced but unusable: ") + blocker;
      return ULYSSES_A2A_ERR_UNSUPPORTED;
    }
    path = ULYSSES_A2A_PATH_TMA;
  } else if (forced_path == ULYSSES_A2A_PATH_VEC || forced_path == ULYSSES_A2A_PATH_STAGED) {
    path = ULYSSES_A2A_PATH_VEC;  // the staged path is decided with the vector width below
  } else {
    path = blocker ? ULYSSES_A2A_PATH_VEC : ULYSSES_A2A_PATH_TMA;
    if (path == ULYSSES_A2A_PATH_TMA && payload / (chunked ? B : 1) <= kVecSmallLaunchBytes)
      path = ULYSSES_A2A_PATH_VEC;  // small launches: the vector kernel's latency is lower
  }

  // sequence rows per work unit; a small vector launch gets smaller units so
  // that about two per SM exist
  int64_t unit_target = path == ULYSSES_A2A_PATH_TMA ? kTmaTileTargetBytes : kTileTargetBytes;
  if (path == ULYSSES_A2A_PATH_VEC) {
    const int64_t spread = payload / (chunked ? B : 1) / (2 * (int64_t)num_sms);
    if (spread < unit_target) unit_target = spread > kVecMinTileBytes ? spread : kVecMinTileBytes;
  }
  int64_t rows = unit_target / row_bytes;
  if (tune.rows_per_tile > 0) rows = tune.rows_per_tile;
  if (rows < 1) rows = 1;
  if (rows > kTmaMaxBoxDim) rows = kTmaMaxBoxDim;
  if (path == ULYSSES_A2A_PATH_TMA) {
    while (rows > 1 && rows * row_bytes > kTmaMaxTileBytes) --rows;
  }
  if (rows > S) rows = S;

  const int64_t T = (S + rows - 1) / rows;  // ceil-div: the ragged last tile is a unit too
  const int64_t nb = chunked ? 1 : B;
  const int64_t blocks_wide = (only_out >= 0 ? (int64_t)w : (int64_t)w * w) * ntensors;
  int64_t units;
  if (mul_overflows(blocks_wide, nb, &tmp) || mul_overflows(tmp, T, &units)) {
    set_err(err, "unit count overflows");
    return ULYSSES_A2A_ERR_INVALID;
  }

  p->path = path;
  p->row_bytes = row_bytes;
  p->rows_per_tile = rows;
  p->tiles_per_block = T;
  p->tail_rows = S % rows;
  p->units = units;
  p->payload_bytes = only_out >= 0 ? slab_bytes * ntensors : payload;
  p->launches = chunked ? (int32_t)(B > INT32_MAX ? INT32_MAX : B) : 1;
  p->row_pitch = pitch;
  p->order = tune.order >= 0 ? (tune.order ? 1 : 0) : kDefaultOrder;

  if (path == ULYSSES_A2A_PATH_TMA) {
    const int64_t tile_bytes = rows * row_bytes;
    const int64_t stage_bytes = (tile_bytes + 1023) / 1024 * 1024;
    const bool persistent = tune.chunk_units == 0;
    const int ctas = tune.ctas_per_sm > 0 ? tune.ctas_per_sm : kTmaDefaultCtasPerSm;
    // Producer warps per CTA, each with a sub-ring of sp stages. A requested
    // total stage count is split evenly over the producers.
    int np;
    if (tune.producers > 0) {
      np = tune.producers;
    } else if (persistent) {
      np = kTmaDefaultProducers;
    } else {
      np = 1;
    }
    const int min_sp = persistent ? 2 : 1;
    int64_t sp = 0;
    for (; np >= 1; --np) {
      sp = tune.stages > 0 ? tune.stages / np : (persistent ? kTmaStagesPerProducer : 1);
      const int64_t budget = (tune.stages > 0 || !persistent) ? kTmaSmemMax : kTmaSmemBudget;
      while (sp > min_sp && np * sp * stage_bytes > budget) --sp;
      if (sp >= min_sp && np * sp <= kTmaMaxStages && np * sp * stage_bytes <= kTmaSmemMax) break;
    }
    if (np < 1) {
      // cannot hold the tiles: let the VEC path take it (or fail if forced)
      if (forced_path == ULYSSES_A2A_PATH_TMA) {
        set_err(err, "TMA ring of %lld-byte tiles does not fit shared memory", tile_bytes);
        return ULYSSES_A2A_ERR_UNSUPPORTED;
      }
      p->path = path = ULYSSES_A2A_PATH_VEC;
    } else {
      p->producers = np;
      p->stages = (int32_t)(np * sp);
      // half of each sub-ring loads ahead, the other half lets stores drain;
      // a one-stage ring (L = S = 1) loads, stores, and waits for the store
      // to read its stage before the next load
      int64_t look = tune.lookahead > 0 ? tune.lookahead : sp - sp / 2;
      if (look > sp - 1) look = sp - 1;
      if (look < 1) look = 1;
      p->lookahead = (int32_t)look;
      p->smem_bytes = np * sp * stage_bytes;
      p->block = 32 * np;
      if (persistent) {
        p->chunk_units = 0;
        int64_t g = (int64_t)num_sms * ctas;
        p->grid = (int32_t)(units < g ? units : g);
      } else {
        int64_t chunk = tune.chunk_units > 0 ? tune.chunk_units : np;
        // keep the grid within the launch limit on huge problems
        if ((units + chunk - 1) / chunk > INT32_MAX) chunk = (units + INT32_MAX - 1) / INT32_MAX;
        if (chunk > INT32_MAX) {
          set_err(err, "%lld units cannot be scheduled", units);
          return ULYSSES_A2A_ERR_UNSUPPORTED;
        }
        p->chunk_units = (int32_t)chunk;
        p->grid = (int32_t)((units + chunk - 1) / chunk);
        // Residency cap: reserve enough shared memory per CTA that at most
        // `cap` CTAs fit on an SM, which bounds the bytes in flight per SM.
        int64_t cap = tune.ctas_per_sm;
        if (cap <= 0) {
          const int64_t per_cta_inflight = np * tile_bytes;
          cap = (kTmaInflightPerSm + per_cta_inflight / 2) / per_cta_inflight;
          if (cap < 1) cap = 1;
          if (cap > 32) cap = 32;
        }
        {
          int64_t per_cta = (kSmemPerSm / cap - kSmemReservedPerCta) / 1024 * 1024;
          if (per_cta > kTmaSmemMax) per_cta = kTmaSmemMax;
          if (per_cta > p->smem_bytes) p->smem_bytes = per_cta;
        }
      }
      p->vec_bytes = 16;
    }
  }
  if (path == ULYSSES_A2A_PATH_VEC) {
    int v = 16;
    while (v > 1) {
      bool ok = (row_bytes % v) == 0 && ((pitch * E) % v) == 0;
      for (int k = 0; k < nin && ok; ++k) ok = (reinterpret_cast<uintptr_t>(in[k]) % v) == 0;
      for (int k = 0; k < nout && ok; ++k)
        ok = !used_out(k) || (reinterpret_cast<uintptr_t>(out[k]) % v) == 0;
      if (ok) break;
      v >>= 1;
    }
    if (units >= (int64_t(1) << 31)) {
      set_err(err, "%lld work units exceed the VEC path's 2^31 limit", units);
      return ULYSSES_A2A_ERR_UNSUPPORTED;
    }
    if (rows * (row_bytes / v) >= (int64_t(1) << 31)) {
      set_err(err, "one VEC tile exceeds 2^31 vectors");
      return ULYSSES_A2A_ERR_UNSUPPORTED;
    }
    // one CTA per unit (units < 2^31 was checked above), or a grid-stride
    // grid of ctas_per_sm CTAs per SM when that knob is set
    int64_t g = tune.ctas_per_sm > 0 ? (int64_t)num_sms * tune.ctas_per_sm : units;
    // Runs that start at one offset past a 16-byte boundary on each side move
    // as 16-byte destination vectors between a peeled head and tail: straight
    // when the two offsets are equal (peeled = 1), each vector joined from two
    // aligned source vectors when they differ (peeled = 2). Not one-output
    // launches, whose inputs are other ranks' windows.
    int a_in = 0, a_out = 0;
    const bool sides = v < 16 && only_out < 0 && forced_path != ULYSSES_A2A_PATH_STAGED &&
                       row_bytes >= kPeelMinRunBytes &&
                       side_offsets(in, nin, out, nout, row_bytes, pitch * E, &a_in, &a_out);
    const int peeled = !sides ? 0 : (a_in == a_out ? 1 : 2);
    p->vec_bytes = peeled ? 16 : v;
    p->peeled = peeled;
    p->stages = 0;
    p->lookahead = 0;
    p->producers = 0;
    p->smem_bytes = 0;
    p->block = kVecBlock;
    p->grid = (int32_t)(units < g ? units : g);

    // The staged path's fixed-phase form takes a dense [B, S, H, D] side whose
    // gathered slabs share one offset past a 16-byte boundary, in pieces of at
    // most 8 bytes, when enough threads can move strided chunks (unless the
    // per-piece form is asked for).
    const int ng = w * ntensors;
    const int64_t HDE = row_bytes * ng;
    bool fixed_phase = tune.staged_form == 0 && pitch * E == HDE && v <= 8 &&
                       phase_movers(HDE) >= kPhaseMinMovers;
    {
      const void* const* gs = mode == 0 ? const_cast<const void* const*>(out) : in;
      for (int k = 1; k < ng && fixed_phase; ++k)
        fixed_phase = (reinterpret_cast<uintptr_t>(gs[k]) & 15u) ==
                      (reinterpret_cast<uintptr_t>(gs[0]) & 15u);
    }
    // The re-aligning path takes what the vector path could only move in
    // pieces of kStageMaxPiece bytes or less, and 8-byte-granular runs that
    // the fixed-phase form takes, or what it is forced onto, except
    // one-output launches.
    const bool forced_stage = forced_path == ULYSSES_A2A_PATH_STAGED;
    const bool auto_stage = forced_path == ULYSSES_A2A_PATH_AUTO && !peeled && only_out < 0 &&
                            (v <= kStageMaxPiece || (v == 8 && fixed_phase));
    if (forced_stage || auto_stage) {
      StageGeometry sg;
      if (stage_geometry(row_bytes, ng, S, tune.rows_per_tile, &sg, fixed_phase,
                         fixed_phase && mode == 0 && v >= 4)) {
        const int64_t nbl = chunked ? 1 : B;
        int64_t su;
        if (mul_overflows((int64_t)w * nbl, sg.tiles, &su) || su >= (int64_t(1) << 31)) {
          set_err(err, "%lld staged work units exceed the 2^31 limit", su);
          return ULYSSES_A2A_ERR_UNSUPPORTED;
        }
        // one short-lived CTA per unit (the hardware hands them to SMs as they
        // free up), or a grid-stride grid of ctas_per_sm CTAs per SM
        const int64_t sgrid = tune.ctas_per_sm > 0 ? (int64_t)num_sms * tune.ctas_per_sm : su;
        p->path = ULYSSES_A2A_PATH_STAGED;
        p->fixed_phase = fixed_phase ? 1 : 0;
        p->rows_per_tile = sg.rows;
        p->tiles_per_block = sg.tiles;
        p->tail_rows = S % sg.rows;
        p->units = su;
        p->smem_bytes = sg.smem_bytes;
        p->block = kStageBlock;
        p->grid = (int32_t)(su < sgrid ? su : sgrid);
      } else if (forced_stage) {
        set_err(err, "staged path forced but one row of %lld bytes does not fit its shared memory",
                row_bytes * w * ntensors);
        return ULYSSES_A2A_ERR_UNSUPPORTED;
      }
    }
  }
  return ULYSSES_A2A_OK;
}

}  // namespace ua2a
