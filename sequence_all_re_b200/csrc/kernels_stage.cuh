// kernels_stage.cuh - the re-aligning copy path of the Ulysses 4D all-to-all
// re-layout: 16-byte global loads and stores for shapes whose runs or base
// addresses are not 16-byte aligned, with the realignment done in shared
// memory.
//
// Same element map as the other paths (FastVideo API docs, device_communicators/
// ulysses_a2a, `run_armed`): mode 0 out_r[b, j*S_local + s, h', d] =
// x_j[b, s, r*(H/w) + h', d]; mode 1 is its inverse.
//
// A work unit is (b, j, t): S_tile rows s0.. of plane b of the strided slab j
// ([B, S_local, H, D] side, rows P bytes apart, the first HDE = ng * R bytes of
// each row belonging to the slab) together with the matching row range of all
// ng gathered slabs g ([B, S_local*w, H/w, D] side, one contiguous range of
// rows * R bytes each, at sequence offset j*S_local + s0). Here R = (H/w)*D*E
// is one run and ng the head groups of a strided row (w, or T*w for T
// head-packed tensors; gathered slab g holds head group g).
//
// The strided side of a unit is one contiguous segment of rows * HDE bytes
// when the slab is dense (P == HDE), else one segment of HDE bytes per row.
//
// Shared memory holds the unit in gathered order: region g (RS bytes apart)
// holds gathered range g, placed at an offset whose value mod 16 equals the
// range's global address mod 16. So:
//   * the gathered side moves as aligned 16-byte vectors between global and
//     shared memory (only the first and last chunk of a range may be partial);
//   * the strided side moves as aligned 16-byte global vectors too, each one
//     split into (or assembled from) G-byte pieces at their places in the
//     regions, where G (1..16) is the largest power of two dividing R, P and
//     every slab base address, so that every piece is G-aligned on both sides;
//     a chunk whose 16 bytes land contiguously in one region moves as aligned
//     shared-memory words instead.
// Mode 0: strided rows -> regions (phase A), regions -> gathered ranges (B).
// Mode 1: gathered ranges -> regions (phase A), regions -> strided rows (B).
// Global bytes outside the unit are never read or written: a partial chunk
// moves only its valid G-byte pieces.
#pragma once

#include <cstdint>

#include "kernels_vec.cuh"  // FastDiv, fdiv, streaming load/store helpers, PDL switch
#include "ulysses_a2a.h"

namespace ua2a {

struct StageParams {
  const char* in[ULYSSES_A2A_MAX_W];
  char* out[ULYSSES_A2A_MAX_W];
  int64_t S_local;
  int64_t b0;             // first plane of this launch
  int64_t P;              // bytes between rows (b, s), (b, s+1) of the strided side
  int32_t R;              // bytes of one run, (H/w)*D*E
  int32_t HDE;            // slab bytes of one strided row, ng * R
  int32_t w;              // sequence blocks (j)
  int32_t ng;             // head groups per strided row, and gathered slabs
  int32_t rows_per_tile;  // S_tile
  uint32_t units;         // nb * w * T
  uint32_t tile0;         // first tile of each (b, j) block in this launch
  int32_t RS;             // bytes per region in shared memory (a multiple of 16)
  int32_t Cs;             // 16-byte chunks scanned per strided row: (HDE + 30) / 16
  int32_t Cg;             // 16-byte chunks scanned per gathered range: (S_tile*R + 30) / 16
  FastDiv div_T;          // tiles per (b, j) block in this launch
  FastDiv div_w;
  FastDiv div_R;
  FastDiv div_ng;
  FastDiv div_Cs;
  FastDiv div_Cg;
};

template <int G>
struct PieceOf;
template <> struct PieceOf<1> { using type = unsigned char; };
template <> struct PieceOf<2> { using type = unsigned short; };
template <> struct PieceOf<4> { using type = unsigned int; };
template <> struct PieceOf<8> { using type = unsigned long long; };
template <> struct PieceOf<16> { using type = uint4; };

template <int G>
union Chunk16 {
  uint4 v;
  typename PieceOf<G>::type e[16 / G];
};

// Bytes [x0, x1) of the aligned 16-byte global chunk at h, as G-byte loads
// (the other bytes of the result are zero and never used).
template <int G>
__device__ __forceinline__ uint4 load_pieces(const char* h, int x0, int x1) {
  using PT = typename PieceOf<G>::type;
  Chunk16<G> c;
  c.v = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int k = 0; k < 16 / G; ++k)
    if (k * G >= x0 && k * G < x1) c.e[k] = ld_stream(reinterpret_cast<const PT*>(h + k * G));
  return c.v;
}

template <int G>
__device__ __forceinline__ void store_pieces(char* h, const uint4& v, int x0, int x1) {
  using PT = typename PieceOf<G>::type;
  Chunk16<G> c;
  c.v = v;
#pragma unroll
  for (int k = 0; k < 16 / G; ++k)
    if (k * G >= x0 && k * G < x1) st_stream(reinterpret_cast<PT*>(h + k * G), c.e[k]);
}

// The pieces [x0, x1) of one strided-side chunk whose byte 0 lies o0 bytes
// after the start of a strided segment beginning at unit row i0 (a segment is
// one row, or all the unit's rows when they are contiguous). Piece x holds the
// segment's byte o = o0 + x: with q = o / R, byte col = o % R of head group
// g = q % ng of unit row i = i0 + q / ng, which lives in region g at row i.
// STORE = true writes the pieces of v into the regions (mode 0), false reads
// them from the regions into the result (mode 1).
template <int G, bool STORE>
__device__ __forceinline__ uint4 strided_pieces(unsigned char* sm, const int32_t* rbase,
                                                const StageParams& p, uint4 v, int x0, int x1,
                                                int32_t o0, int32_t i0) {
  using PT = typename PieceOf<G>::type;
  Chunk16<G> c;
  c.v = v;
  const uint32_t q = fdiv((uint32_t)(o0 + x0), p.div_R);
  const uint32_t di = fdiv(q, p.div_ng);
  int32_t g = (int32_t)(q - di * (uint32_t)p.ng);
  int32_t col = o0 + x0 - (int32_t)q * p.R;
  int32_t iR = (i0 + (int32_t)di) * p.R;
  int32_t at = rbase[g] + iR + col;
#pragma unroll
  for (int k = 0; k < 16 / G; ++k) {
    const int x = k * G;
    if (x >= x0 && x < x1) {
      PT* s = reinterpret_cast<PT*>(sm + at);
      if (STORE)
        *s = c.e[k];
      else
        c.e[k] = *s;
      col += G;
      at += G;
      if (col == p.R && x + G < x1) {  // the next piece starts the next head group
        col = 0;
        if (++g == p.ng) {             // ... of the next row
          g = 0;
          iR += p.R;
        }
        at = rbase[g] + iR;
      }
    }
  }
  return c.v;
}

// A whole 16-byte chunk to / from 16 consecutive bytes of shared memory at
// byte offset `at` (which must be even): one 16-, two 8- or four 4-byte accesses
// when `at` allows them, else (at = 2 mod 4) a 2-byte access, three 4-byte
// accesses 2 bytes into the chunk (their words assembled with byte
// permutes: bytes 2..5 of the chunk are the upper half of word 0 and the
// lower half of word 1, and so on) and a final 2-byte access.
__device__ __forceinline__ void smem_put16(unsigned char* sm, int32_t at, const uint4& v) {
  unsigned char* d = sm + at;
  if ((at & 15) == 0) {
    *reinterpret_cast<uint4*>(d) = v;
  } else if ((at & 7) == 0) {
    reinterpret_cast<uint2*>(d)[0] = make_uint2(v.x, v.y);
    reinterpret_cast<uint2*>(d)[1] = make_uint2(v.z, v.w);
  } else if ((at & 3) == 0) {
    uint32_t* q = reinterpret_cast<uint32_t*>(d);
    q[0] = v.x;
    q[1] = v.y;
    q[2] = v.z;
    q[3] = v.w;
  } else {
    *reinterpret_cast<unsigned short*>(d) = (unsigned short)v.x;
    *reinterpret_cast<uint32_t*>(d + 2) = __byte_perm(v.x, v.y, 0x5432);
    *reinterpret_cast<uint32_t*>(d + 6) = __byte_perm(v.y, v.z, 0x5432);
    *reinterpret_cast<uint32_t*>(d + 10) = __byte_perm(v.z, v.w, 0x5432);
    *reinterpret_cast<unsigned short*>(d + 14) = (unsigned short)(v.w >> 16);
  }
}

__device__ __forceinline__ uint4 smem_get16(const unsigned char* sm, int32_t at) {
  const unsigned char* d = sm + at;
  if ((at & 15) == 0) return *reinterpret_cast<const uint4*>(d);
  uint4 v;
  if ((at & 7) == 0) {
    const uint2 a = reinterpret_cast<const uint2*>(d)[0];
    const uint2 b = reinterpret_cast<const uint2*>(d)[1];
    v = make_uint4(a.x, a.y, b.x, b.y);
  } else if ((at & 3) == 0) {
    const uint32_t* q = reinterpret_cast<const uint32_t*>(d);
    v = make_uint4(q[0], q[1], q[2], q[3]);
  } else {
    const uint32_t h0 = *reinterpret_cast<const unsigned short*>(d);
    const uint32_t m1 = *reinterpret_cast<const uint32_t*>(d + 2);
    const uint32_t m2 = *reinterpret_cast<const uint32_t*>(d + 6);
    const uint32_t m3 = *reinterpret_cast<const uint32_t*>(d + 10);
    const uint32_t h4 = *reinterpret_cast<const unsigned short*>(d + 14);
    v = make_uint4(__byte_perm(h0, m1, 0x5410), __byte_perm(m1, m2, 0x5432),
                   __byte_perm(m2, m3, 0x5432), __byte_perm(m3, h4, 0x5432));
  }
  return v;
}

// The same pieces for a whole chunk (x0 = 0, x1 = 16, so o0 >= 0) when a run
// is at least 16 bytes long: the chunk then meets at most one head-group
// boundary, lim bytes in, and byte x goes to at1 + x before it and to
// at2 + x after it.
template <int G, bool STORE>
__device__ __forceinline__ uint4 strided_pieces_full(unsigned char* sm, const int32_t* rbase,
                                                     const StageParams& p, uint4 v, int32_t o0,
                                                     int32_t i0) {
  using PT = typename PieceOf<G>::type;
  Chunk16<G> c;
  c.v = v;
  const uint32_t q = fdiv((uint32_t)o0, p.div_R);
  const uint32_t di = fdiv(q, p.div_ng);
  int32_t g = (int32_t)(q - di * (uint32_t)p.ng);
  const int32_t col = o0 - (int32_t)q * p.R;
  int32_t iR = (i0 + (int32_t)di) * p.R;
  const int32_t at1 = rbase[g] + iR + col;
  const int32_t lim = p.R - col;  // bytes before the next head group
  if (G >= 2 && lim >= 16) {      // the whole chunk lands contiguously (at1 is even)
    if (STORE) {
      smem_put16(sm, at1, c.v);
      return c.v;
    }
    return smem_get16(sm, at1);
  }
  int32_t at2 = at1;
  if (lim < 16) {
    if (++g == p.ng) {            // the next head group starts the next row
      g = 0;
      iR += p.R;
    }
    at2 = rbase[g] + iR - lim;
  }
#pragma unroll
  for (int k = 0; k < 16 / G; ++k) {
    const int x = k * G;
    PT* s = reinterpret_cast<PT*>(sm + (x < lim ? at1 : at2) + x);
    if (STORE)
      *s = c.e[k];
    else
      c.e[k] = *s;
  }
  return c.v;
}

// Loads in flight per thread before they are placed in shared memory.
constexpr int kStageUnroll = 4;
// 256-thread CTAs; at least 4 resident per SM.
constexpr int kStageMinBlocksPerSm = 4;

template <int G, int MODE>
__global__ void __launch_bounds__(256, kStageMinBlocksPerSm)
    ua2a_stage_kernel(const __grid_constant__ StageParams p) {
  extern __shared__ __align__(16) unsigned char sm[];
  int32_t* rbase = reinterpret_cast<int32_t*>(sm + (size_t)p.ng * p.RS);
#if UA2A_PDL
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
  const int32_t R = p.R;
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
    const int32_t L = rows * R;  // bytes of each gathered range of this unit
    // byte offset of the unit's range in every gathered slab, and of its first
    // row in strided slab j
    const int64_t goff = ((b * p.w + j) * p.S_local + s0) * (int64_t)R;
    const int64_t soff = (b * p.S_local + s0) * p.P;
    const char* srow0 = (MODE == 0 ? p.in[j] : p.out[j]) + soff;
    // Strided segments: the unit's rows are one contiguous segment when the
    // slab is dense (P == HDE), else one segment per row.
    const bool dense = p.P == (int64_t)p.HDE;
    const int32_t seg_len = dense ? rows * p.HDE : p.HDE;
    const int32_t nS = dense ? (int32_t)(((reinterpret_cast<uintptr_t>(srow0) & 15u) + seg_len + 15) >> 4)
                             : rows * p.Cs;

    for (int g = threadIdx.x; g < p.ng; g += blockDim.x) {
      const char* ga = (MODE == 0 ? p.out[g] : p.in[g]) + goff;
      rbase[g] = g * p.RS + (int32_t)(reinterpret_cast<uintptr_t>(ga) & 15u);
    }
    __syncthreads();

    if (MODE == 0) {
      // phase A: strided rows -> regions, kStageUnroll loads in flight per thread
      const int32_t nA = nS;
      for (int32_t e0 = threadIdx.x; e0 < nA; e0 += blockDim.x * kStageUnroll) {
        uint4 v[kStageUnroll];
#pragma unroll
        for (int k = 0; k < kStageUnroll; ++k) {
          const int32_t e = e0 + k * (int32_t)blockDim.x;
          if (e < nA) {
            const uint32_t i = dense ? 0u : fdiv((uint32_t)e, p.div_Cs);
            const int32_t c = dense ? e : e - (int32_t)i * p.Cs;
            const char* a = srow0 + (int64_t)i * p.P;
            const int32_t o0 = 16 * c - (int32_t)(reinterpret_cast<uintptr_t>(a) & 15u);
            const int x0 = o0 < 0 ? -o0 : 0;
            const int x1 = seg_len - o0 < 16 ? seg_len - o0 : 16;
            if (x0 == 0 && x1 == 16)
              v[k] = ld_stream(reinterpret_cast<const uint4*>(a + o0));
            else if (x0 < x1)
              v[k] = load_pieces<G>(a + o0, x0, x1);
          }
        }
#pragma unroll
        for (int k = 0; k < kStageUnroll; ++k) {
          const int32_t e = e0 + k * (int32_t)blockDim.x;
          if (e < nA) {
            const uint32_t i = dense ? 0u : fdiv((uint32_t)e, p.div_Cs);
            const int32_t c = dense ? e : e - (int32_t)i * p.Cs;
            const char* a = srow0 + (int64_t)i * p.P;
            const int32_t o0 = 16 * c - (int32_t)(reinterpret_cast<uintptr_t>(a) & 15u);
            const int x0 = o0 < 0 ? -o0 : 0;
            const int x1 = seg_len - o0 < 16 ? seg_len - o0 : 16;
            if (x0 == 0 && x1 == 16 && p.R >= 16)
              strided_pieces_full<G, true>(sm, rbase, p, v[k], o0, (int32_t)i);
            else if (x0 < x1)
              strided_pieces<G, true>(sm, rbase, p, v[k], x0, x1, o0, (int32_t)i);
          }
        }
      }
      __syncthreads();
      // phase B: regions -> gathered ranges (aligned in both)
      const int32_t nB = p.ng * p.Cg;
      for (int32_t e = threadIdx.x; e < nB; e += blockDim.x) {
        const uint32_t g = fdiv((uint32_t)e, p.div_Cg);
        const int32_t c = e - (int32_t)g * p.Cg;
        char* d = p.out[g] + goff;
        const int32_t o0 = 16 * c - (int32_t)(reinterpret_cast<uintptr_t>(d) & 15u);
        const int x0 = o0 < 0 ? -o0 : 0;
        const int x1 = L - o0 < 16 ? L - o0 : 16;
        if (x0 >= x1) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(sm + (int32_t)g * p.RS + 16 * c);
        if (x0 == 0 && x1 == 16)
          st_stream(reinterpret_cast<uint4*>(d + o0), v);
        else
          store_pieces<G>(d + o0, v, x0, x1);
      }
    } else {
      // phase A: gathered ranges -> regions, kStageUnroll loads in flight per thread
      const int32_t nA = p.ng * p.Cg;
      for (int32_t e0 = threadIdx.x; e0 < nA; e0 += blockDim.x * kStageUnroll) {
        uint4 v[kStageUnroll];
#pragma unroll
        for (int k = 0; k < kStageUnroll; ++k) {
          const int32_t e = e0 + k * (int32_t)blockDim.x;
          if (e < nA) {
            const uint32_t g = fdiv((uint32_t)e, p.div_Cg);
            const int32_t c = e - (int32_t)g * p.Cg;
            const char* s = p.in[g] + goff;
            const int32_t o0 = 16 * c - (int32_t)(reinterpret_cast<uintptr_t>(s) & 15u);
            const int x0 = o0 < 0 ? -o0 : 0;
            const int x1 = L - o0 < 16 ? L - o0 : 16;
            if (x0 == 0 && x1 == 16)
              v[k] = ld_stream(reinterpret_cast<const uint4*>(s + o0));
            else if (x0 < x1)
              v[k] = load_pieces<G>(s + o0, x0, x1);
          }
        }
#pragma unroll
        for (int k = 0; k < kStageUnroll; ++k) {
          const int32_t e = e0 + k * (int32_t)blockDim.x;
          if (e < nA) {
            const uint32_t g = fdiv((uint32_t)e, p.div_Cg);
            const int32_t c = e - (int32_t)g * p.Cg;
            const char* s = p.in[g] + goff;
            const int32_t o0 = 16 * c - (int32_t)(reinterpret_cast<uintptr_t>(s) & 15u);
            const int x0 = o0 < 0 ? -o0 : 0;
            const int x1 = L - o0 < 16 ? L - o0 : 16;
            // the region mirrors the range's alignment, so chunk c sits whole
            // at region offset 16c; a partial chunk fills only its valid pieces
            unsigned char* slot = sm + (int32_t)g * p.RS + 16 * c;
            if (x0 == 0 && x1 == 16) {
              *reinterpret_cast<uint4*>(slot) = v[k];
            } else if (x0 < x1) {
              Chunk16<G> cv;
              cv.v = v[k];
#pragma unroll
              for (int m = 0; m < 16 / G; ++m)
                if (m * G >= x0 && m * G < x1)
                  *reinterpret_cast<typename PieceOf<G>::type*>(slot + m * G) = cv.e[m];
            }
          }
        }
      }
      __syncthreads();
      // phase B: regions -> strided rows
      const int32_t nB = nS;
      for (int32_t e = threadIdx.x; e < nB; e += blockDim.x) {
        const uint32_t i = dense ? 0u : fdiv((uint32_t)e, p.div_Cs);
        const int32_t c = dense ? e : e - (int32_t)i * p.Cs;
        char* a = const_cast<char*>(srow0) + (int64_t)i * p.P;
        const int32_t o0 = 16 * c - (int32_t)(reinterpret_cast<uintptr_t>(a) & 15u);
        const int x0 = o0 < 0 ? -o0 : 0;
        const int x1 = seg_len - o0 < 16 ? seg_len - o0 : 16;
        if (x0 >= x1) continue;
        if (x0 == 0 && x1 == 16) {
          const uint4 v = p.R >= 16 ? strided_pieces_full<G, false>(sm, rbase, p,
                                                                    make_uint4(0, 0, 0, 0), o0,
                                                                    (int32_t)i)
                                    : strided_pieces<G, false>(sm, rbase, p, make_uint4(0, 0, 0, 0),
                                                               0, 16, o0, (int32_t)i);
          st_stream(reinterpret_cast<uint4*>(a + o0), v);
        } else {
          const uint4 v = strided_pieces<G, false>(sm, rbase, p, make_uint4(0, 0, 0, 0), x0, x1,
                                                   o0, (int32_t)i);
          store_pieces<G>(a + o0, v, x0, x1);
        }
      }
    }
    __syncthreads();  // the regions are reused by the next unit
  }
}

}  // namespace ua2a
