// kernels_phase.cuh - fixed-phase form of the re-aligning copy path of the
// Ulysses 4D all-to-all re-layout, for shapes whose [B, S_local, H, D] side is
// dense (rows HDE = ng * R bytes apart) and whose gathered slabs all start the
// same number of bytes past a 16-byte boundary.
//
// Element map as on the other paths (FastVideo API docs, device_communicators/
// ulysses_a2a, `run_armed`): mode 0 out_r[b, j*S_local + s, h', d] =
// x_j[b, s, r*(H/w) + h', d]; mode 1 is its inverse.
//
// Units, regions and the gathered side are those of the staged kernel
// (kernels_stage.cuh): unit (b, j, t) is S_tile rows s0.. of plane b of strided
// slab j with the matching row range of every gathered slab g (R = (H/w)*D*E
// bytes per row and slab, ng gathered slabs: w, or T*w for T head-packed
// tensors). Shared memory holds ng regions RS bytes apart; region g holds
// range g starting a_g bytes in, a_g being the ranges' common address mod 16,
// so the gathered side moves as aligned 16-byte vectors.
//
// The strided side of a unit is one contiguous segment of rows * HDE bytes,
// moved as aligned 16-byte global chunks as well. Chunk c holds segment bytes
// o .. o + 15 with o = 16c - a_s (a_s: the segment's address mod 16); byte o
// is byte o mod R of run q = o / R, that is of head group q mod ng in row
// q / ng, which region g = q mod ng holds at a_g + (q / ng) * R + o mod R.
// Relative to row i0 = floor(o / HDE), the shared-memory places of a chunk's
// 16 / G pieces (G bytes each, G dividing R, HDE and every base address)
// depend only on o mod HDE. Thread t takes the chunks c = t + m * nthr, with
// nthr a multiple of HDE / gcd(HDE, 16): 16 * nthr is then a multiple of HDE,
// every chunk of the thread has the same o mod HDE, and chunk m starts
// step_rows = 16 * nthr / HDE rows after chunk m - 1. So a thread works out
// its piece offsets once per unit, and a piece costs one add and one shared
// access.
//
// Mode 1: gathered ranges -> regions by cp.async in two commit groups (A),
// pieces from the regions -> strided chunks (B), the first half of the unit's
// rows assembled while the second group is in flight.
// Mode 0, pieces of 2 bytes or less (scatter form): strided chunks -> pieces
// into the regions (A, loads held in registers), regions -> gathered ranges
// (B). Mode 0, pieces of 4 or 8 bytes (gather form): the strided segment lands
// by cp.async in a swizzled image (no regions), in two commit groups, and
// threads build whole gathered chunks from it, each thread's chunks sharing
// one phase within a run (the same offset argument, with period
// R / gcd(R, 16) chunks).
// Global bytes outside the unit are never read or written: a partial chunk at
// either end of a range or segment moves only its valid pieces.
#pragma once

#include <cstdint>

#include "kernels_stage.cuh"  // PieceOf, Chunk16, load_pieces, store_pieces
#include "kernels_vec.cuh"    // FastDiv, fdiv, streaming load/store helpers, PDL switch
#include "ulysses_a2a.h"

namespace ua2a {

struct PhaseParams {
  const char* in[ULYSSES_A2A_MAX_W];
  char* out[ULYSSES_A2A_MAX_W];
  int64_t S_local;
  int64_t b0;             // first plane of this launch
  int32_t R;              // bytes of one run, (H/w)*D*E
  int32_t HDE;            // bytes of one strided row, ng * R (dense)
  int32_t w;              // sequence blocks (j)
  int32_t ng;             // head groups per strided row, and gathered slabs
  int32_t rows_per_tile;  // S_tile
  uint32_t units;         // nb * w * T
  uint32_t tile0;         // first tile of each (b, j) block in this launch
  int32_t RS;             // bytes per region in shared memory (a multiple of 16)
  int32_t Cg;             // 16-byte chunks scanned per gathered range: (S_tile*R + 30) / 16
  int32_t nthr;           // threads moving strided chunks, a multiple of HDE / gcd(HDE, 16)
  int32_t step_rows;      // 16 * nthr / HDE
  FastDiv div_T;          // tiles per (b, j) block in this launch
  FastDiv div_w;
  FastDiv div_R;
  FastDiv div_HDE;
  FastDiv div_Cg;
  FastDiv div_ng;
  // mode 0: threads that build gathered chunks (a multiple of R / gcd(R, 16)),
  // and the region chunk count padded to such a multiple
  int32_t nthr0;
  int32_t Cpad;
  FastDiv div_Cpad;
};

// Mode 0 keeps the strided segment in shared memory as loaded, its 16-byte
// chunks permuted within each 128-byte block: byte x sits at swz(x). Bits 4-6
// are XORed with bits 9-11, which spreads one warp's piece accesses (16*ng
// bytes apart in the segment) over the banks.
__device__ __forceinline__ int32_t swz(int32_t x) { return x ^ (((x >> 9) & 7) << 4); }

// Strided chunks in flight per thread in mode 0 (2 with 1-byte pieces, whose
// 16 offsets leave no registers for more). Measured on B200 against 6 and 8
// at 4 CTAs per SM (64 registers; 8 spills): 4 at 5 CTAs per SM is fastest
// on every shape but 8-byte runs (6-byte runs 0.81 against 0.79 and 0.64).
constexpr int kPhaseUnroll = 4;

// Shared-memory offsets of the 16 / G pieces of a strided chunk whose byte 0
// is byte kap (0 <= kap < HDE) of a strided row, from that row's place in
// region 0: piece n is byte col of the run of head group g in row dr (0 or
// later) of the regions.
template <int G>
__device__ __forceinline__ void piece_offsets(int32_t (&off)[16 / G], int32_t kap, int32_t R,
                                              int32_t RS, int32_t ng, const FastDiv& div_R) {
  int32_t g = (int32_t)fdiv((uint32_t)kap, div_R);
  int32_t col = kap - g * R;
  int32_t dr = 0;
#pragma unroll
  for (int n = 0; n < 16 / G; ++n) {
    off[n] = g * RS + dr * R + col;
    col += G;
    if (col == R) {  // the next piece starts the next run
      col = 0;
      if (++g == ng) {
        g = 0;
        ++dr;
      }
    }
  }
}

// Asynchronous 16-byte copy global -> shared (cp.async, cached in L2 only):
// the data goes to shared memory without passing through registers, so a
// thread can have all its chunks of a unit in flight at once. Both
// addresses must be 16-byte aligned.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Bytes [x0, x1) of the aligned 16-byte global chunk at h as G-byte loads
// cached in L2 with the normal policy, as cp.async.cg caches the whole chunks
// beside them: a partial chunk shares its 32-byte sector with a neighbour that
// cp.async reads, and an evict-first load would let that sector leave L2 in
// between (the other bytes of the result are zero and never used).
template <int G>
__device__ __forceinline__ uint4 load_pieces_l2(const char* h, int x0, int x1) {
  using PT = typename PieceOf<G>::type;
  Chunk16<G> c;
  c.v = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int k = 0; k < 16 / G; ++k)
    if (k * G >= x0 && k * G < x1) c.e[k] = __ldcg(reinterpret_cast<const PT*>(h + k * G));
  return c.v;
}

// Wait until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 256-thread CTAs; at least 5 resident per SM (4 with 1-byte pieces, whose
// mode-1 instance spills at 48 registers).
constexpr int kPhaseMinBlocksPerSm = 5;

template <int G, int MODE>
__global__ void __launch_bounds__(256, G == 1 ? 4 : kPhaseMinBlocksPerSm)
    ua2a_phase_kernel(const __grid_constant__ PhaseParams p) {
  using PT = typename PieceOf<G>::type;
  constexpr int NP = 16 / G;  // pieces per chunk
  extern __shared__ __align__(16) unsigned char sm[];
#if UA2A_PDL
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
  const int32_t R = p.R;
  const int32_t HDE = p.HDE;
  const int32_t RS = p.RS;
  const int32_t tid = (int32_t)threadIdx.x;
  for (uint32_t u = blockIdx.x; u < p.units; u += gridDim.x) {
    // u = (b_rel * w + j) * T + t
    const uint32_t q = fdiv(u, p.div_T);
    const uint32_t t = u - q * p.div_T.d;
    const uint32_t bl = fdiv(q, p.div_w);
    const uint32_t j = q - bl * p.div_w.d;
    const int64_t b = p.b0 + bl;
    const int64_t s0 = (int64_t)(p.tile0 + t) * p.rows_per_tile;
    const int64_t left = p.S_local - s0;
    const int32_t rows = (int32_t)(left < p.rows_per_tile ? left : p.rows_per_tile);
    const int32_t L = rows * R;      // bytes of each gathered range of this unit
    const int32_t segB = rows * HDE;  // bytes of the strided segment
    // the unit's range in every gathered slab, and its segment of strided slab j
    const int64_t goff = ((b * p.w + j) * p.S_local + s0) * (int64_t)R;
    const uintptr_t seg = reinterpret_cast<uintptr_t>(MODE == 0 ? p.in[j] : p.out[j]) +
                          (uintptr_t)((b * p.S_local + s0) * (int64_t)HDE);
    const int32_t a_s = (int32_t)(seg & 15u);
    const int32_t a_g =
        (int32_t)((reinterpret_cast<uintptr_t>(MODE == 0 ? p.out[0] : p.in[0]) + (uintptr_t)goff) & 15u);
    char* const seg16 = reinterpret_cast<char*>(seg - (uintptr_t)a_s);  // 16-byte aligned
    const int32_t nS = (a_s + segB + 15) >> 4;  // strided chunks of the segment

    // This thread's strided chunks c = tid + m * nthr: the row i0 of its first
    // chunk's byte 0 (o may be negative, o >= -15, so i0 >= -1 - 15 / HDE) and
    // its phase kap = o - i0 * HDE. Chunk m's pieces sit at
    // base0 + m * dbase + off[n] (>= 0 for every piece inside the segment).
    const int32_t o_first = 16 * tid - a_s;
    const int32_t i0 = (int32_t)fdiv((uint32_t)(o_first + 16 * HDE), p.div_HDE) - 16;
    const int32_t kap = o_first - i0 * HDE;
    const int32_t base0 = a_g + i0 * R;
    const int32_t dbase = p.step_rows * R;
    const bool mover = tid < p.nthr;
    int32_t off[NP];

    if constexpr (MODE == 0 && G >= 4) {
      // Pieces of 4 bytes or more: gather form.
      // phase A: the strided segment's chunks land by cp.async in the
      // swizzled image, in two commit groups: those holding the unit's first
      // rowsA rows (c < cI1) first.
      const int32_t rowsA = rows >> 1;
      const int32_t cI1 = (a_s + rowsA * HDE + 15) >> 4;
      {
        bool first_open = true;
        for (int32_t c = tid; c < nS; c += (int32_t)blockDim.x) {
          if (first_open && c >= cI1) {
            cp_async_commit();
            first_open = false;
          }
          const int32_t o = 16 * c - a_s;
          unsigned char* dst = sm + swz(16 * c);
          if (o >= 0 && segB - o >= 16) {
            cp_async16(dst, seg16 + 16 * c);
          } else {  // a partial chunk at either end of the segment: its valid pieces
            const int x0 = o < 0 ? -o : 0;
            const int x1 = segB - o < 16 ? segB - o : 16;
            Chunk16<G> cv;
            cv.v = load_pieces_l2<G>(seg16 + 16 * c, x0, x1);
#pragma unroll
            for (int n = 0; n < NP; ++n)
              if (n * G >= x0 && n * G < x1) *reinterpret_cast<PT*>(dst + n * G) = cv.e[n];
          }
        }
        if (first_open) cp_async_commit();
        cp_async_commit();
      }
      // phase B: gathered chunks built from the image and stored. Thread tid
      // takes chunks e = tid + m * nthr0 of the ng regions laid end to end,
      // Cpad chunks each; chunk c of region g holds region bytes
      // q = 16c - a_g .. q + 15, byte q being byte q mod R of row q / R of
      // head group g, segment byte (q / R) * HDE + g * R + q mod R. All of a
      // thread's chunks share q mod R, so the segment offsets of its pieces
      // from row q0 / R, group g are one list.
      const int32_t r_n = (a_g + L + 15) >> 4;        // chunks holding range bytes
      const int32_t cB1 = (a_g + rowsA * R) >> 4;     // chunks inside the first rowsA rows
      const bool mover0 = tid < p.nthr0;
      if (mover0) {
        const int32_t q = 16 * tid - a_g + 16 * R;    // >= 0, same phase as 16 * tid - a_g
        int32_t col = q - (int32_t)fdiv((uint32_t)q, p.div_R) * R;
        int32_t drow = 0;
#pragma unroll
        for (int n = 0; n < NP; ++n) {
          off[n] = drow * HDE + col;
          col += G;
          if (col == R) {
            col = 0;
            ++drow;
          }
        }
      }
      auto build = [&](int32_t e, bool first) {
        const int32_t g = (int32_t)fdiv((uint32_t)e, p.div_Cpad);
        const int32_t c = e - g * p.Cpad;
        if (c >= r_n || (c < cB1) != first) return;
        const int32_t q0 = 16 * c - a_g;
        const int32_t i0 = (int32_t)fdiv((uint32_t)(q0 + 16 * R), p.div_R) - 16;  // floor(q0 / R)
        const int32_t base = a_s + i0 * HDE + g * R;
        char* d = p.out[g] + (goff + q0);
        Chunk16<G> cv;
        if (q0 >= 0 && L - q0 >= 16) {
#pragma unroll
          for (int n = 0; n < NP; ++n) cv.e[n] = *reinterpret_cast<const PT*>(sm + swz(base + off[n]));
          st_stream(reinterpret_cast<uint4*>(d), cv.v);
        } else {
          const int x0 = q0 < 0 ? -q0 : 0;
          const int x1 = L - q0 < 16 ? L - q0 : 16;
          cv.v = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int n = 0; n < NP; ++n)
            if (n * G >= x0 && n * G < x1) cv.e[n] = *reinterpret_cast<const PT*>(sm + swz(base + off[n]));
          store_pieces<G>(d, cv.v, x0, x1);
        }
      };
      const int32_t nE = p.ng * p.Cpad;
      cp_async_wait<1>();
      __syncthreads();
      if (mover0)
        for (int32_t e = tid; e < nE; e += p.nthr0) build(e, true);
      cp_async_wait<0>();
      __syncthreads();
      if (mover0)
        for (int32_t e = tid; e < nE; e += p.nthr0) build(e, false);
    } else if constexpr (MODE == 0) {
      // Pieces of 2 bytes or less: scatter form.
      // phase A: strided chunks -> regions, U loads in flight
      constexpr int U = G == 1 ? 2 : kPhaseUnroll;
      if (mover) {
        piece_offsets<G>(off, kap, R, RS, p.ng, p.div_R);
        for (int32_t m0 = 0; tid + m0 * p.nthr < nS; m0 += U) {
          uint4 v[U];
#pragma unroll
          for (int k = 0; k < U; ++k) {
            const int32_t c = tid + (m0 + k) * p.nthr;
            if (c < nS) {
              const int32_t o = 16 * c - a_s;
              const int x0 = o < 0 ? -o : 0;
              const int x1 = segB - o < 16 ? segB - o : 16;
              if (x0 == 0 && x1 == 16)
                v[k] = ld_stream(reinterpret_cast<const uint4*>(seg16 + 16 * c));
              else
                v[k] = load_pieces<G>(seg16 + 16 * c, x0, x1);
            }
          }
#pragma unroll
          for (int k = 0; k < U; ++k) {
            const int32_t c = tid + (m0 + k) * p.nthr;
            if (c < nS) {
              const int32_t o = 16 * c - a_s;
              const int x0 = o < 0 ? -o : 0;
              const int x1 = segB - o < 16 ? segB - o : 16;
              const int32_t at = base0 + (m0 + k) * dbase;
              Chunk16<G> cv;
              cv.v = v[k];
              if (x0 == 0 && x1 == 16) {
#pragma unroll
                for (int n = 0; n < NP; ++n) *reinterpret_cast<PT*>(sm + (at + off[n])) = cv.e[n];
              } else {
#pragma unroll
                for (int n = 0; n < NP; ++n)
                  if (n * G >= x0 && n * G < x1) *reinterpret_cast<PT*>(sm + (at + off[n])) = cv.e[n];
              }
            }
          }
        }
      }
      __syncthreads();
      // phase B: regions -> gathered ranges, aligned on both sides
      const int32_t nB = p.ng * p.Cg;
      for (int32_t e = tid; e < nB; e += (int32_t)blockDim.x) {
        const int32_t g = (int32_t)fdiv((uint32_t)e, p.div_Cg);
        const int32_t c = e - g * p.Cg;
        const int32_t o0 = 16 * c - a_g;
        const int x0 = o0 < 0 ? -o0 : 0;
        const int x1 = L - o0 < 16 ? L - o0 : 16;
        if (x0 >= x1) continue;
        char* d = p.out[g] + (goff + o0);
        const uint4 v = *reinterpret_cast<const uint4*>(sm + (g * RS + 16 * c));
        if (x0 == 0 && x1 == 16)
          st_stream(reinterpret_cast<uint4*>(d), v);
        else
          store_pieces<G>(d, v, x0, x1);
      }
    } else {
      // phase A: gathered ranges -> regions by cp.async, numbered region-
      // fastest (e = c * ng + g), so that each thread issues the chunks
      // holding the unit's first rowsA rows (c < cgA) before the rest: two
      // commit groups. The strided chunks inside those rows (c < cA) are
      // assembled while the second group is still in flight.
      const int32_t rowsA = rows >> 1;
      const int32_t cgA = (a_g + rowsA * R + 15) >> 4;
      const int32_t cA = (a_s + rowsA * HDE) >> 4;
      // Blocks of 8 chunks (128 bytes) of one region, regions fastest:
      // e = (cb * ng + g) * 8 + k moves chunk c = cb * 8 + k of region g; the
      // first group takes whole blocks up to cgA8 >= cgA.
      const int32_t cgA8 = (cgA + 7) & ~7;
      const int32_t nA = p.ng * ((p.Cg + 7) & ~7);
      bool first_open = true;
      for (int32_t e = tid; e < nA; e += (int32_t)blockDim.x) {
        const int32_t q = e >> 3;
        const int32_t cb = (int32_t)fdiv((uint32_t)q, p.div_ng);
        const int32_t g = q - cb * p.ng;
        const int32_t c = cb * 8 + (e & 7);
        if (first_open && c >= cgA8) {
          cp_async_commit();
          first_open = false;
        }
        if (c >= p.Cg) continue;
        const int32_t o0 = 16 * c - a_g;
        const int x0 = o0 < 0 ? -o0 : 0;
        const int x1 = L - o0 < 16 ? L - o0 : 16;
        if (x0 >= x1) continue;
        const char* src = p.in[g] + (goff + o0);
        unsigned char* slot = sm + (g * RS + 16 * c);
        if (x0 == 0 && x1 == 16) {
          cp_async16(slot, src);
        } else {  // a partial chunk at either end of a range: its valid pieces
          Chunk16<G> cv;
          cv.v = load_pieces_l2<G>(src, x0, x1);
#pragma unroll
          for (int n = 0; n < NP; ++n)
            if (n * G >= x0 && n * G < x1) *reinterpret_cast<PT*>(slot + n * G) = cv.e[n];
        }
      }
      if (first_open) cp_async_commit();
      cp_async_commit();
      // phase B: pieces from the regions -> strided chunks, first those of
      // the first rowsA rows, then (once every copy has landed) the rest
      auto gather = [&](int32_t c, int32_t m) {
        const int32_t o = 16 * c - a_s;
        const int x0 = o < 0 ? -o : 0;
        const int x1 = segB - o < 16 ? segB - o : 16;
        const int32_t at = base0 + m * dbase;
        Chunk16<G> cv;
        if (x0 == 0 && x1 == 16) {
#pragma unroll
          for (int n = 0; n < NP; ++n) cv.e[n] = *reinterpret_cast<const PT*>(sm + (at + off[n]));
          st_stream(reinterpret_cast<uint4*>(seg16 + 16 * c), cv.v);
        } else {
          cv.v = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int n = 0; n < NP; ++n)
            if (n * G >= x0 && n * G < x1) cv.e[n] = *reinterpret_cast<const PT*>(sm + (at + off[n]));
          store_pieces<G>(seg16 + 16 * c, cv.v, x0, x1);
        }
      };
      cp_async_wait<1>();
      __syncthreads();
      int32_t m = 0;
      if (mover) {
        piece_offsets<G>(off, kap, R, RS, p.ng, p.div_R);
        for (; tid + m * p.nthr < cA; ++m) gather(tid + m * p.nthr, m);
      }
      cp_async_wait<0>();
      __syncthreads();
      if (mover)
        for (; tid + m * p.nthr < nS; ++m) gather(tid + m * p.nthr, m);
    }
    __syncthreads();  // the regions are reused by the next unit
  }
}

}  // namespace ua2a
