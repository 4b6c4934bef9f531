// kernels_peel.cuh - the vector path's peeled and shifted kernels of the
// Ulysses 4D all-to-all re-layout (FastVideo API docs, device_communicators/
// ulysses_a2a, `run_armed`: mode 0 out_r[b, j*S_local + s, h', d] =
// x_j[b, s, r*(H/w) + h', d], mode 1 its inverse), for runs that start off a
// 16-byte boundary. Same launch parameters, units and CTAs as the
// whole-vector kernel of kernels_vec.cuh.
//
// Peeled variant (ua2a_peel_kernel): when every slab starts the same number
// of bytes a past a 16-byte boundary and runs and rows are whole multiples of
// 16 bytes, every run on either side starts a bytes past a boundary. The
// whole-vector kernel could then only move 2-byte pieces (for a = 2), yet each
// run is 16 - a head bytes, then L*E/16 - 1 aligned 16-byte vectors, then a
// tail bytes, at the same offsets on both sides. The peeled kernel moves the
// vectors as the whole-vector kernel does (shifted by the head), and each
// run's head and tail in aligned pieces of 8, 4, 2 and 1 bytes held in the
// same registers, all of a thread's loads in flight before its stores.
//
// Shifted variant (ua2a_shift_kernel): the source slabs share one offset a_s
// and the destination slabs another, a_d. Each run's destination is then
// split as above by a_d, and the 16 source bytes of a destination vector lie
// d = a_s - a_d (mod 16) bytes into an aligned 32-byte source window: two
// aligned 16-byte loads joined by funnel shifts. Every aligned load holds at
// least one byte the copy needs, so none leaves the 16-byte granules its
// slab occupies.
#pragma once

#include <cstdint>

#include "kernels_vec.cuh"

namespace ua2a {

// Aligned pieces of bytes [x0, x1) of a 16-byte window, x0 = 0 or x1 = 16: a
// run's head (x0 = its start offset, x1 = 16) or its tail (x0 = 0, x1 = the
// tail's length). They split into at most one piece each of 8, 4, 2 and 1
// bytes, whose offsets follow from the binary digits of x0 (head) or x1 (tail).
struct WindowPieces {
  uint32_t o8, o4, o2, o1;  // offsets in the window
  bool f8, f4, f2, f1;      // which pieces exist
};

__device__ __forceinline__ WindowPieces window_pieces(uint32_t x0, uint32_t x1) {
  WindowPieces w;
  if (x0 > 0) {  // head: climb from x0 to 16 in growing aligned pieces
    uint32_t q = x0;
    w.f1 = q & 1; w.o1 = q; q += w.f1 ? 1 : 0;
    w.f2 = q & 2; w.o2 = q; q += w.f2 ? 2 : 0;
    w.f4 = q & 4; w.o4 = q; q += w.f4 ? 4 : 0;
    w.f8 = q & 8; w.o8 = q;
  } else {       // tail: [0, x1) in shrinking pieces
    w.f8 = x1 & 8; w.o8 = 0;
    w.f4 = x1 & 4; w.o4 = x1 & 8;
    w.f2 = x1 & 2; w.o2 = x1 & 12;
    w.f1 = x1 & 1; w.o1 = x1 & 14;
  }
  return w;
}

// The pieces of one partial window, packed in four registers: the 8-byte
// piece in x, y, the 4-byte in z, the 2- and 1-byte in w (store_pieces takes
// them back from there).
__device__ __forceinline__ uint4 load_pieces(const char* win, const WindowPieces& pc) {
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (pc.f8) {
    const uint2 t = ld_stream(reinterpret_cast<const uint2*>(win + pc.o8));
    v.x = t.x;
    v.y = t.y;
  }
  if (pc.f4) v.z = ld_stream(reinterpret_cast<const unsigned int*>(win + pc.o4));
  if (pc.f2) v.w = ld_stream(reinterpret_cast<const unsigned short*>(win + pc.o2));
  if (pc.f1) v.w |= (uint32_t)ld_stream(reinterpret_cast<const unsigned char*>(win + pc.o1)) << 16;
  return v;
}

__device__ __forceinline__ void store_pieces(char* win, const WindowPieces& pc, uint4 v) {
  if (pc.f8) st_stream(reinterpret_cast<uint2*>(win + pc.o8), make_uint2(v.x, v.y));
  if (pc.f4) st_stream(reinterpret_cast<unsigned int*>(win + pc.o4), v.z);
  if (pc.f2) st_stream(reinterpret_cast<unsigned short*>(win + pc.o2), (unsigned short)(v.w & 0xFFFFu));
  if (pc.f1) st_stream(reinterpret_cast<unsigned char*>(win + pc.o1), (unsigned char)(v.w >> 16));
}

// The peeled variant (see the top of this file). p.nv = whole vectors per
// run (L*E/16 - 1), p.srow in 16-byte vectors, p.head = 16 - a. A unit's
// index space is its rows' whole vectors, then two edge items per row (the
// run's head, then its tail), so the edge pieces of a unit are in flight with
// its vectors and their 32-byte sectors, shared with the neighbouring vectors,
// are read from DRAM once. A unit whose vectors would not be 16-byte aligned
// on both sides is not touched (the host picks this kernel only when every
// slab starts a bytes past a boundary and runs and rows are 16-byte multiples).
// Resident CTAs per SM the peeled kernel's launch bound asks for, and its
// items per thread (build-time switches). More bytes in flight lose here, as
// on the TMA path: slab bases 2 bytes off, 4 items at 6 CTAs per SM: 0.96 /
// 0.94 of the copy bandwidth; 6 at 5: 0.87 / 0.86; 8 at 4: 0.79 / 0.79.
#ifndef UA2A_PEEL_MIN_BLOCKS
#define UA2A_PEEL_MIN_BLOCKS 6
#endif
#ifndef UA2A_PEEL_ITEMS
#define UA2A_PEEL_ITEMS 4
#endif

template <int MODE, int U>
__global__ void __launch_bounds__(256, UA2A_PEEL_MIN_BLOCKS)
    ua2a_peel_kernel(const __grid_constant__ VecParams p) {
#if UA2A_PDL
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
  const int64_t run = p.run;
  const uint32_t nv = (uint32_t)p.nv;
  const uint32_t nrun = (uint32_t)(run >> 4);  // 16-byte vectors between gathered rows
  const int64_t strided_row = p.srow;          // 16-byte vectors between strided rows
  const uint32_t a = 16u - (uint32_t)p.head;   // run start past its 16-byte boundary
  const uint32_t step = blockDim.x * U;
  for (uint32_t u = blockIdx.x; u < p.units; u += gridDim.x) {
    const VecUnit x = vec_unit(p, u);
    // first run of the unit, from its start (the vectors begin `head` bytes in)
    const int64_t soff = (x.b * p.S_local + x.s0) * strided_row * 16 + (int64_t)x.r * run;
    const int64_t goff = ((x.b * p.w + x.j) * p.S_local + x.s0) * run;
    const char* sb = MODE == 0 ? p.in[x.j] + soff : p.in[x.r] + goff;
    char* db = MODE == 0 ? p.out[x.r] + goff : p.out[x.j] + soff;
    if (((((uintptr_t)sb + p.head) | ((uintptr_t)db + p.head)) & 15) != 0) continue;
    const int64_t src_row = MODE == 0 ? strided_row : (int64_t)nrun;  // in vectors
    const int64_t dst_row = MODE == 0 ? (int64_t)nrun : strided_row;
    const uint4* src = reinterpret_cast<const uint4*>(sb + p.head);
    uint4* dst = reinterpret_cast<uint4*>(db + p.head);
    const uint32_t nvec = (uint32_t)(x.rows * nv);
    const uint32_t n = nvec + 2u * (uint32_t)x.rows;
    for (uint32_t base = threadIdx.x; base < n; base += step) {
      uint4 v[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const uint32_t e = base + k * blockDim.x;
        if (e < nvec) {
          const uint32_t row = fdiv(e, p.div_nv);
          const uint32_t c = e - row * nv;
          v[k] = ld_stream(src + (int64_t)row * src_row + c);
        } else if (e < n) {
          // head: window src[row*src_row] - 16, bytes [a, 16); tail: window
          // src[row*src_row + nv], bytes [0, a)
          const uint32_t i = e - nvec;
          const char* w = reinterpret_cast<const char*>(src + (int64_t)(i >> 1) * src_row +
                                                        ((i & 1) ? nv : 0)) - ((i & 1) ? 0 : 16);
          v[k] = load_pieces(w, (i & 1) ? window_pieces(0, a) : window_pieces(a, 16));
        }
      }
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const uint32_t e = base + k * blockDim.x;
        if (e < nvec) {
          const uint32_t row = fdiv(e, p.div_nv);
          const uint32_t c = e - row * nv;
          st_stream(dst + (int64_t)row * dst_row + c, v[k]);
        } else if (e < n) {
          const uint32_t i = e - nvec;
          char* w = reinterpret_cast<char*>(dst + (int64_t)(i >> 1) * dst_row + ((i & 1) ? nv : 0)) -
                    ((i & 1) ? 0 : 16);
          store_pieces(w, (i & 1) ? window_pieces(0, a) : window_pieces(a, 16), v[k]);
        }
      }
    }
  }
}

// Word i (0..3) of v.
__device__ __forceinline__ uint32_t word_of(const uint4& v, uint32_t i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// The pieces of a window held at their own byte positions in v (byte x of the
// window in byte x of v, as a funnel shift leaves them), stored at win. Every
// piece is aligned to its size, so it lies within one word, or two for the
// 8-byte piece.
__device__ __forceinline__ void store_window_pieces(char* win, const WindowPieces& pc, const uint4& v) {
  if (pc.f8)
    st_stream(reinterpret_cast<uint2*>(win + pc.o8),
              make_uint2(word_of(v, pc.o8 >> 2), word_of(v, (pc.o8 >> 2) + 1)));
  if (pc.f4) st_stream(reinterpret_cast<unsigned int*>(win + pc.o4), word_of(v, pc.o4 >> 2));
  if (pc.f2)
    st_stream(reinterpret_cast<unsigned short*>(win + pc.o2),
              (unsigned short)(word_of(v, pc.o2 >> 2) >> (8 * (pc.o2 & 3))));
  if (pc.f1)
    st_stream(reinterpret_cast<unsigned char*>(win + pc.o1),
              (unsigned char)(word_of(v, pc.o1 >> 2) >> (8 * (pc.o1 & 3))));
}

// Bytes d .. d + 15 of the 32 bytes a, b (a first), for d = 4*Q + sh/8:
// word i of the result is the funnel shift of words Q + i, Q + i + 1.
template <int Q>
__device__ __forceinline__ uint4 funnel16(const uint4& a, const uint4& b, uint32_t sh) {
  const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  return make_uint4(__funnelshift_r(u[Q], u[Q + 1], sh), __funnelshift_r(u[Q + 1], u[Q + 2], sh),
                    __funnelshift_r(u[Q + 2], u[Q + 3], sh), __funnelshift_r(u[Q + 3], u[Q + 4], sh));
}

// The shifted variant (see the top of this file). p.nv = whole destination
// vectors per run (L*E/16, less one when a_d > 0), p.srow in 16-byte vectors,
// p.head = (16 - a_d) mod 16, p.shift = d = 4*Q + r. A unit's index space is
// its rows' destination vectors, then (a_d > 0) two edge items per row: the
// destination head window (bytes [a_d, 16)) and tail window ([0, a_d)). Item
// k of row i draws on the aligned source window at the same place d bytes
// earlier; an edge loads only the halves of its window holding needed bytes.
// A unit whose aligned addresses do not line up is not touched (the host
// picks this kernel only when every slab on each side shares that side's
// offset and runs and rows are 16-byte multiples).
// Items per thread in flight (two loads each) and resident CTAs per SM the
// launch bound asks for (build-time switches). 4 items at 5 CTAs per SM (up to
// 51 registers) keep 80 KB of distinct source vectors in flight per SM; 2 at 6
// kept 48 KB and left the kernel waiting on memory (slab bases 2 bytes off on
// one side: 0.91 / 0.88 of the copy bandwidth against 1.00 / 0.94; 3 at 5:
// 1.01 / 0.93; 4 at 4: 0.92 / 0.87).
#ifndef UA2A_SHIFT_ITEMS
#define UA2A_SHIFT_ITEMS 4
#endif
#ifndef UA2A_SHIFT_MIN_BLOCKS
#define UA2A_SHIFT_MIN_BLOCKS 5
#endif

template <int MODE, int Q>
__global__ void __launch_bounds__(256, UA2A_SHIFT_MIN_BLOCKS)
    ua2a_shift_kernel(const __grid_constant__ VecParams p) {
#if UA2A_PDL
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
  constexpr int U = UA2A_SHIFT_ITEMS;
  const int64_t run = p.run;
  const uint32_t nv = (uint32_t)p.nv;
  const uint32_t nrun = (uint32_t)(run >> 4);
  const int64_t strided_row = p.srow;
  const uint32_t ad = (16u - (uint32_t)p.head) & 15u;  // destination run start past its boundary
  const uint32_t d = (uint32_t)p.shift;
  const uint32_t sh = 8u * (d & 3u);
  const uint32_t nedge = ad ? 2u : 0u;
  const uint32_t step = blockDim.x * U;
  for (uint32_t u = blockIdx.x; u < p.units; u += gridDim.x) {
    const VecUnit x = vec_unit(p, u);
    const int64_t soff = (x.b * p.S_local + x.s0) * strided_row * 16 + (int64_t)x.r * run;
    const int64_t goff = ((x.b * p.w + x.j) * p.S_local + x.s0) * run;
    const char* sb = MODE == 0 ? p.in[x.j] + soff : p.in[x.r] + goff;
    char* db = MODE == 0 ? p.out[x.r] + goff : p.out[x.j] + soff;
    // first destination vector of row 0 and its aligned source window
    const char* sa = sb + p.head - (int32_t)d;
    char* da = db + p.head;
    if (((((uintptr_t)sa) | ((uintptr_t)da)) & 15) != 0) continue;
    const int64_t src_row = MODE == 0 ? strided_row : (int64_t)nrun;  // in vectors
    const int64_t dst_row = MODE == 0 ? (int64_t)nrun : strided_row;
    const uint4* src = reinterpret_cast<const uint4*>(sa);
    uint4* dst = reinterpret_cast<uint4*>(da);
    const uint32_t nvec = (uint32_t)(x.rows * nv);
    const uint32_t n = nvec + nedge * (uint32_t)x.rows;
    for (uint32_t base = threadIdx.x; base < n; base += step) {
      uint4 v0[U], v1[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const uint32_t e = base + k * blockDim.x;
        v0[k] = make_uint4(0u, 0u, 0u, 0u);
        v1[k] = v0[k];
        if (e < nvec) {
          const uint32_t row = fdiv(e, p.div_nv);
          const uint32_t c = e - row * nv;
          const uint4* w = src + (int64_t)row * src_row + c;
          v0[k] = ld_stream(w);
          v1[k] = ld_stream(w + 1);
        } else if (e < n) {
          // head: the window before the row's first vector, destination bytes
          // [ad, 16) <- window bytes [d + ad, d + 16); tail: the window after
          // its last vector, [0, ad) <- [d, d + ad)
          const uint32_t i = e - nvec;
          const bool tail = i & 1;
          const uint4* w = src + (int64_t)(i >> 1) * src_row + (tail ? (int64_t)nv : -1);
          if (tail ? true : d + ad < 16u) v0[k] = ld_stream(w);
          if (tail ? d + ad > 16u : true) v1[k] = ld_stream(w + 1);
        }
      }
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const uint32_t e = base + k * blockDim.x;
        if (e < nvec) {
          const uint32_t row = fdiv(e, p.div_nv);
          const uint32_t c = e - row * nv;
          st_stream(dst + (int64_t)row * dst_row + c, funnel16<Q>(v0[k], v1[k], sh));
        } else if (e < n) {
          const uint32_t i = e - nvec;
          const bool tail = i & 1;
          char* w = reinterpret_cast<char*>(dst + (int64_t)(i >> 1) * dst_row + (tail ? (int64_t)nv : -1));
          store_window_pieces(w, tail ? window_pieces(0, ad) : window_pieces(ad, 16),
                              funnel16<Q>(v0[k], v1[k], sh));
        }
      }
    }
  }
}

}  // namespace ua2a
