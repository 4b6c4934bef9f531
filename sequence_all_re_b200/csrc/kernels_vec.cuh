// kernels_vec.cuh - vectorised LDG/STG copy path of the Ulysses 4D all-to-all
// re-layout (any shape, any alignment).
//
// Mode 0 (FastVideo API docs, device_communicators/ulysses_a2a, `run_armed`,
// mode-0 branch): out_r[b, j*S_local + s, h', d] = x_j[b, s, r*(H/w) + h', d].
// Mode 1 (the else branch, the inverse): out_j[b, s, r*(H/w) + h', d] =
// x_r[b, j*S_local + s, h', d].
//
// For fixed (r, b, j) the (h', d) pairs of one sequence row form a contiguous
// run of L = (H/w)*D elements on BOTH sides, so the copy moves whole runs:
// vectors of V bytes (16 when every base address and the run length allow it,
// otherwise 8/4/2/1), with `ld.global.cs` / `st.global.cs` (streaming, evict
// first: every byte is touched exactly once). A CTA owns one work unit at a
// time: up to S_tile rows of one (r, b, j) block, the last tile of a block
// holding only the S_local % S_tile remaining rows (ceil-div tiling, clamped
// row count). Each thread keeps U vectors in flight before storing them.
//
// A launch may cover every output slab or only one rank's: r in
// {r0 + k*r_stride : k < nr} and j in [j0, j0 + nj). One rank's share of a
// multi-GPU exchange writes its own output slab (one per tensor when T
// tensors are head-packed: head groups t*w + rank, r_stride = w) and reads
// every rank's published input through peer mappings.
#pragma once

#include <cstdint>

#include "ulysses_a2a.h"

// Programmatic dependent launch (see kernels_tma.cuh); 0 turns it off.
#ifndef UA2A_PDL
#define UA2A_PDL 1
#endif

namespace ua2a {

// Division by a run-time invariant divisor d (1 <= d < 2^31) for dividends
// n < 2^31, by multiply-high and shift: the round-up method of Granlund and
// Montgomery, "Division by invariant integers using multiplication" (PLDI 1994).
// With s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1, the quotient is
// (umulhi(n, m) + n) >> s.
struct FastDiv {
  uint32_t d = 1, m = 1, s = 0;
  FastDiv() = default;
  explicit FastDiv(uint32_t div) : d(div) {
    s = 0;
    while ((uint64_t(1) << s) < div) ++s;
    m = (uint32_t)((((uint64_t(1) << s) - div) << 32) / div + 1);
  }
};

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (__umulhi(n, f.m) + n) >> f.s;
}

struct VecParams {
  const char* in[ULYSSES_A2A_MAX_W];
  char* out[ULYSSES_A2A_MAX_W];
  int64_t S_local;
  int64_t b0;            // first plane of this launch
  int64_t nv;            // vectors per run: L*E / V (peeled: whole vectors a run
                         // holds between its head and tail, L*E/16 - 1)
  int64_t srow;          // vectors between rows (b, s), (b, s+1) of the [B,S,H,D] side
  int32_t w;
  int32_t rows_per_tile;
  uint32_t units;        // nr * nb * nj * T
  int32_t order;         // unit numbering: 0 = r outermost, 1 = r innermost
  uint32_t tile0;        // first tile of each (r, b, j) block in this launch
  uint32_t r0, j0;       // first r and first j this launch covers
  uint32_t r_stride;     // head groups between consecutive r of the launch (1, or w to
                         // take one rank's group of each of T head-packed tensors)
  FastDiv div_T;         // tiles per (r, b, j) block in this launch
  FastDiv div_nr;        // r values covered (w, or 1 for one output slab)
  FastDiv div_nj;        // j values covered
  FastDiv div_nb;        // planes in this launch
  FastDiv div_nv;
  // Fields of peeled launches only. They stay last: placed before w, they cost
  // the 8-byte mode-0 whole-vector kernel 8 registers (40 instead of 32), and
  // with them two of its eight resident CTAs per SM.
  int64_t run;           // bytes per run, L*E
  int32_t head;          // bytes before a run's first 16-byte boundary (on the
                         // destination side)
  int32_t shift;         // shifted launches: source offset minus destination
                         // offset past their 16-byte boundaries, mod 16 (1..15)
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) { return __ldcs(p); }
__device__ __forceinline__ uint2 ld_stream(const uint2* p) { return __ldcs(p); }
__device__ __forceinline__ unsigned int ld_stream(const unsigned int* p) { return __ldcs(p); }
__device__ __forceinline__ unsigned short ld_stream(const unsigned short* p) { return __ldcs(p); }
__device__ __forceinline__ unsigned char ld_stream(const unsigned char* p) { return __ldcs(p); }
__device__ __forceinline__ unsigned long long ld_stream(const unsigned long long* p) {
  return __ldcs(p);
}
__device__ __forceinline__ void st_stream(uint4* p, uint4 v) { __stcs(p, v); }
__device__ __forceinline__ void st_stream(uint2* p, uint2 v) { __stcs(p, v); }
__device__ __forceinline__ void st_stream(unsigned int* p, unsigned int v) { __stcs(p, v); }
__device__ __forceinline__ void st_stream(unsigned short* p, unsigned short v) { __stcs(p, v); }
__device__ __forceinline__ void st_stream(unsigned char* p, unsigned char v) { __stcs(p, v); }
__device__ __forceinline__ void st_stream(unsigned long long* p, unsigned long long v) {
  __stcs(p, v);
}

// 256-thread CTAs, at least 6 resident per SM: caps the kernel at 40
// registers (75% occupancy). The 16-byte and peeled kernels need that many;
// kernels on vectors of 8 bytes or less fit in 32 registers without spilling,
// so they take 8 per SM (full occupancy: more loads in flight per SM).
constexpr int kVecMinBlocksPerSm = 6;

template <typename V>
constexpr int vec_min_blocks_per_sm() {
  return sizeof(V) == 16 ? kVecMinBlocksPerSm : 8;
}

// Work unit u of a launch -> (r, j, plane b, first row s0, rows).
struct VecUnit {
  uint32_t r, j;
  int64_t b, s0, rows;
};

__device__ __forceinline__ VecUnit vec_unit(const VecParams& p, uint32_t u) {
  uint32_t t, j, r, bl;
  if (p.order == 0) {
    // u = ((r_rel * nb + b_rel) * nj + j_rel) * T + t
    const uint32_t q = fdiv(u, p.div_T);
    t = u - q * p.div_T.d;
    const uint32_t q2 = fdiv(q, p.div_nj);
    j = q - q2 * p.div_nj.d;
    r = fdiv(q2, p.div_nb);
    bl = q2 - r * p.div_nb.d;
  } else {
    // u = ((b_rel * nj + j_rel) * T + t) * nr + r_rel
    const uint32_t q = fdiv(u, p.div_nr);
    r = u - q * p.div_nr.d;
    const uint32_t q2 = fdiv(q, p.div_T);
    t = q - q2 * p.div_T.d;
    bl = fdiv(q2, p.div_nj);
    j = q2 - bl * p.div_nj.d;
  }
  VecUnit x;
  x.r = p.r0 + r * p.r_stride;
  x.j = j + p.j0;
  x.b = p.b0 + bl;
  x.s0 = (int64_t)(p.tile0 + t) * p.rows_per_tile;
  const int64_t rows_left = p.S_local - x.s0;
  x.rows = rows_left < p.rows_per_tile ? rows_left : p.rows_per_tile;
  return x;
}

template <typename V, int MODE, int U>
__global__ void __launch_bounds__(256, vec_min_blocks_per_sm<V>())
    ua2a_vec_kernel(const __grid_constant__ VecParams p) {
#if UA2A_PDL
  // programmatic dependent launch: start the next grid's launch, then wait for
  // the previous one to finish before touching global memory
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
  const uint32_t nv = (uint32_t)p.nv;
  const int64_t strided_row = p.srow;  // vectors between rows s, s+1 of [B,S,H,D] (pitch)
  const uint32_t step = blockDim.x * U;
  for (uint32_t u = blockIdx.x; u < p.units; u += gridDim.x) {
    const VecUnit x = vec_unit(p, u);
    const uint32_t r = x.r, j = x.j;
    const int64_t b = x.b, s0 = x.s0, rows = x.rows;
    // strided side: row (b, s0), head group r; gathered side: row (b, j*S_local + s0)
    const int64_t soff = (b * p.S_local + s0) * strided_row + (int64_t)r * p.nv;
    const int64_t goff = ((b * p.w + j) * p.S_local + s0) * p.nv;
    const V* src;
    V* dst;
    if (MODE == 0) {
      src = reinterpret_cast<const V*>(p.in[j]) + soff;
      dst = reinterpret_cast<V*>(p.out[r]) + goff;
    } else {
      src = reinterpret_cast<const V*>(p.in[r]) + goff;
      dst = reinterpret_cast<V*>(p.out[j]) + soff;
    }
    const uint32_t n = (uint32_t)(rows * p.nv);
    for (uint32_t base = threadIdx.x; base < n; base += step) {
      V v[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const uint32_t e = base + k * blockDim.x;
        if (e < n) {
          const uint32_t row = fdiv(e, p.div_nv);
          const uint32_t c = e - row * nv;
          const int64_t off = (MODE == 0) ? (int64_t)row * strided_row + c : (int64_t)e;
          v[k] = ld_stream(src + off);
        }
      }
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const uint32_t e = base + k * blockDim.x;
        if (e < n) {
          const uint32_t row = fdiv(e, p.div_nv);
          const uint32_t c = e - row * nv;
          const int64_t off = (MODE == 0) ? (int64_t)e : (int64_t)row * strided_row + c;
          st_stream(dst + off, v[k]);
        }
      }
    }
  }
}

}  // namespace ua2a
