// kernels_tma.cuh - TMA bulk-tensor copy path of the Ulysses 4D all-to-all
// re-layout (sm_100a).
//
// Same element map as the VEC path (FastVideo API docs, device_communicators/
// ulysses_a2a, `run_armed`): mode 0 out_r[b, j*S_local+s, h', d] =
// x_j[b, s, r*(H/w)+h', d]; mode 1 is its inverse.
//
// Each rank slab gets one tensor map per side, both with the sequence row
// extent bounded to S_local per plane (never a flattened B*S_local row range,
// so a ragged last tile can neither read the next plane nor write into the
// next rank's block):
//   strided side  [B, S_local, H, D]      4-D map, dims (D, H, S_local, B),
//                                          box (D, H/w, S_tile, 1);
//   gathered side [B, S_local*w, H/w, D]  5-D map, dims (D, H/w, S_local, w, B),
//                                          box (D, H/w, S_tile, 1, 1).
// Both boxes land in shared memory as the same dense [S_tile][H/w][D] image,
// so a tile is moved by one cp.async.bulk.tensor load (completing on an
// mbarrier) and one cp.async.bulk.tensor store from the same stage, with no
// thread touching the data. A tile that runs past S_local is clipped by the
// hardware: the load zero-fills the rows beyond the plane and the store skips
// them. No multicast is used anywhere.
//
// Strided-side maps take the row pitch as their sequence stride, so a slab
// may sit inside wider rows (q, k or v of a packed projection output).
//
// Schedule: one elected thread in each of `producers` warps per CTA drives its
// own ring of `stages` shared-memory tiles over every producers-th unit this
// CTA owns, keeping `lookahead` loads and up to stages - lookahead stores in
// flight. A CTA owns either a chunk of `chunk_units` consecutive units (the
// default, with one producer and one unit per CTA: short-lived single-warp
// CTAs handed out by the hardware as SMs free up, their residency per SM
// capped by the shared memory the planner reserves) or, with chunk_units = 0,
// units blockIdx.x + i*gridDim.x of a persistent grid. Units are numbered with
// the destination rank innermost or outermost (`order`). Launches use
// programmatic dependent launch: each CTA waits for the previous grid before
// touching global memory.
//
// Every mbarrier wait is bounded in time; on expiry the kernel records the
// failure in the context's status word, waits (bounded) for its own copies
// still in flight and returns.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "plan.h"  // shared limits: kTmaMaxStages, kTmaMaxProducers
#include "ulysses_a2a.h"

namespace ua2a {

// Give up an mbarrier wait after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// Status word bits.
constexpr unsigned kStatusWaitTimeout = 1u;
constexpr unsigned kStatusDrainTimeout = 2u;

struct TmaParams {
  CUtensorMap strided[ULYSSES_A2A_MAX_W_TMA];   // slabs laid out [B, S_local, H, D]
  CUtensorMap gathered[ULYSSES_A2A_MAX_W_TMA];  // slabs laid out [B, S_local*w, H/w, D]
  unsigned int* status;                         // [flags, block+1, tile]
  int64_t units;                                // w * nb * w * T
  int32_t w;
  int32_t Hw;                                   // H / w
  int32_t rows_per_tile;                        // S_tile
  int32_t tiles_per_block;                      // tiles per (r, b, j) block in this launch
  int32_t tile0;                                //   ... starting at tile tile0 (0 = whole block)
  int32_t b0;                                   // first plane of this launch
  int32_t nb;                                   // planes in this launch
  uint32_t tile_bytes;                          // full box bytes (clipped rows included)
  uint32_t stage_bytes;                         // tile_bytes rounded up to 1 KB
  int32_t stages;                               // S: shared-memory tiles per producer
  int32_t lookahead;                            // L: loads in flight per producer, 1 <= L < S
  int32_t producers;                            // producer warps per CTA (1..8)
  int32_t order;                                // unit numbering: 0 = r outermost, 1 = r innermost
  int32_t chunk_units;                          // 0 = persistent grid; else units per CTA
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most
// limit_ns of %globaltimer (checked every 256 polls) and at most 2^30 polls.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && global_ns() - t0 > limit_ns) return false;
  }
  return false;
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Every byte is touched once, so the copies may carry an L2 evict-first
// policy (UA2A_CACHE_HINT=1 at build time); by default they carry none.
// The stored tile was written to shared memory by a TMA load (async proxy)
// and is read by a TMA store (async proxy); the mbarrier wait already orders
// the two, so no proxy fence is needed between them (UA2A_STORE_FENCE=1 adds
// one, for measurement).
#ifndef UA2A_STORE_FENCE
#define UA2A_STORE_FENCE 0
#endif

#ifndef UA2A_CACHE_HINT
#define UA2A_CACHE_HINT 0
#endif

// Programmatic dependent launch (launch attribute + griddepcontrol); 0 turns
// it off at build time, for measurement.
#ifndef UA2A_PDL
#define UA2A_PDL 1
#endif

// Let the next grid in the stream begin launching, then wait until every grid
// this one depends on has finished and its memory operations are visible.
// Both are no-ops for a grid launched without the programmatic attribute.
__device__ __forceinline__ void pdl_launch_then_wait() {
#if UA2A_PDL
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol = 0;
#if UA2A_CACHE_HINT
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
#endif
  return pol;
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, uint64_t pol) {
#if UA2A_CACHE_HINT
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(pol)
      : "memory");
#else
  (void)pol;
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
#endif
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4, uint64_t pol) {
#if UA2A_CACHE_HINT
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(c4), "l"(pol)
      : "memory");
#else
  (void)pol;
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(c4)
      : "memory");
#endif
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3, uint64_t pol) {
#if UA2A_CACHE_HINT
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group.L2::cache_hint"
      " [%0, {%2, %3, %4, %5}], [%1], %6;" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(pol)
      : "memory");
#else
  (void)pol;
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group"
      " [%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
#endif
}

__device__ __forceinline__ void tma_store_5d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3, int c4, uint64_t pol) {
#if UA2A_CACHE_HINT
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group.L2::cache_hint"
      " [%0, {%2, %3, %4, %5, %6}], [%1], %7;" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "l"(pol)
      : "memory");
#else
  (void)pol;
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group"
      " [%0, {%2, %3, %4, %5, %6}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
#endif
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// All but the newest N bulk groups have finished READING shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Run-time N (the instruction takes an immediate): 0 <= n < kTmaMaxStages.
__device__ __forceinline__ void bulk_wait_read_n(int n) {
  switch (n) {
    case 0: bulk_wait_read<0>(); break;
    case 1: bulk_wait_read<1>(); break;
    case 2: bulk_wait_read<2>(); break;
    case 3: bulk_wait_read<3>(); break;
    case 4: bulk_wait_read<4>(); break;
    case 5: bulk_wait_read<5>(); break;
    case 6: bulk_wait_read<6>(); break;
    case 7: bulk_wait_read<7>(); break;
    case 8: bulk_wait_read<8>(); break;
    case 9: bulk_wait_read<9>(); break;
    case 10: bulk_wait_read<10>(); break;
    case 11: bulk_wait_read<11>(); break;
    case 12: bulk_wait_read<12>(); break;
    case 13: bulk_wait_read<13>(); break;
    case 14: bulk_wait_read<14>(); break;
    default: bulk_wait_read<0>(); break;   // strictest: every store has read its stage
  }
}

__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

struct UnitCoord {
  int r, b, j, s0;
};

__device__ __forceinline__ UnitCoord decode_unit(const TmaParams& p, int64_t u) {
  UnitCoord c;
  if (p.order == 0) {
    // destination rank outermost: u = ((r * nb + b_rel) * w + j) * T + t
    const int64_t t = u % p.tiles_per_block;
    int64_t q = u / p.tiles_per_block;
    c.j = (int)(q % p.w);
    q /= p.w;
    c.b = p.b0 + (int)(q % p.nb);
    c.r = (int)(q / p.nb);
    c.s0 = (int)((p.tile0 + t) * p.rows_per_tile);
  } else {
    // destination rank innermost: u = ((b_rel * w + j) * T + t) * w + r, so w
    // consecutive units cover whole rows of the [B, S_local, H, D] side
    c.r = (int)(u % p.w);
    int64_t q = u / p.w;
    const int64_t t = q % p.tiles_per_block;
    q /= p.tiles_per_block;
    c.j = (int)(q % p.w);
    c.b = p.b0 + (int)(q / p.w);
    c.s0 = (int)((p.tile0 + t) * p.rows_per_tile);
  }
  return c;
}

template <int MODE>
__global__ void __launch_bounds__(32 * kTmaMaxProducers, 1)
    ua2a_tma_kernel(const __grid_constant__ TmaParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[kTmaMaxStages];
  // One elected lane per warp; warp k is producer k of p.producers.
  if ((threadIdx.x & 31) != 0) return;
  const int k = (int)(threadIdx.x >> 5);
  const int NP = p.producers;

  // The CTA owns units first + i*G (i = 0 .. n_cta-1): either every
  // gridDim.x-th unit (persistent grid, chunk_units = 0) or a contiguous chunk
  // of chunk_units units (G = 1, the hardware hands out chunks as CTAs finish).
  // Producer k takes i = k, k + NP, k + 2*NP, ... as its sequence m = 0 .. n-1.
  int64_t G, first, n_cta;
  if (p.chunk_units > 0) {
    G = 1;
    first = (int64_t)blockIdx.x * p.chunk_units;
    n_cta = p.units - first < p.chunk_units ? p.units - first : p.chunk_units;
  } else {
    G = gridDim.x;
    first = blockIdx.x;
    n_cta = (p.units - first + G - 1) / G;
  }
  if (first >= p.units || k >= NP) return;
  const int64_t n = n_cta > k ? (n_cta - k + NP - 1) / NP : 0;
  const int S = p.stages;      // stages of this producer's sub-ring
  const int L = p.lookahead;   // its loads in flight, 1 <= L < S (L = S = 1 allowed)
  const uint32_t smem0 = smem_addr(smem) + (uint32_t)(k * S) * p.stage_bytes;
  const uint32_t bar0 = smem_addr(full) + 8u * (uint32_t)(k * S);

  const uint64_t pol = l2_evict_first_policy();
  for (int s = 0; s < S; ++s) mbar_init(bar0 + 8u * s, 1);
  fence_barrier_init();
  fence_proxy_async_smem();
  // the previous kernel in the stream may still be running: wait for it
  // before touching global memory (programmatic dependent launch)
  pdl_launch_then_wait();

  auto unit_of = [&](int64_t m) { return first + (k + m * NP) * G; };
  auto issue_load = [&](int64_t m) {
    const int s = (int)(m % S);
    const UnitCoord c = decode_unit(p, unit_of(m));
    const uint32_t bar = bar0 + 8u * s;
    const uint32_t dst = smem0 + (uint32_t)s * p.stage_bytes;
    mbar_arrive_expect_tx(bar, p.tile_bytes);
    if (MODE == 0)
      tma_load_4d(dst, &p.strided[c.j], bar, 0, c.r * p.Hw, c.s0, c.b, pol);
    else
      tma_load_5d(dst, &p.gathered[c.r], bar, 0, 0, c.s0, c.j, c.b, pol);
  };
  auto issue_store = [&](int64_t m) {
    const int s = (int)(m % S);
    const UnitCoord c = decode_unit(p, unit_of(m));
    const uint32_t src = smem0 + (uint32_t)s * p.stage_bytes;
    if (MODE == 0)
      tma_store_5d(&p.gathered[c.r], src, 0, 0, c.s0, c.j, c.b, pol);
    else
      tma_store_4d(&p.strided[c.j], src, 0, c.r * p.Hw, c.s0, c.b, pol);
    bulk_commit();
  };

  // Sub-ring of S stages: tile m lives in stage m % S. L loads run ahead of
  // the tile being stored, so up to S - L stores may still be reading their
  // stages; loading tile m+L needs only the store of tile m+L-S, issued S-L
  // tiles earlier, to have read its stage out. TMA operations issued by one
  // thread complete roughly one at a time, so several producers per CTA keep
  // enough of them in flight.
  const int64_t pre = n < L ? n : L;
  for (int64_t m = 0; m < pre; ++m) issue_load(m);

  for (int64_t m = 0; m < n; ++m) {
    const int s = (int)(m % S);
    const uint32_t parity = (uint32_t)((m / S) & 1);
    if (!mbar_wait_bounded(bar0 + 8u * s, parity)) {
      // Record, then drain: loads m .. issued-1 may still be landing in this
      // CTA's shared memory; wait for each once more (bounded) before leaving.
      atomicOr(p.status, kStatusWaitTimeout);
      atomicExch(p.status + 1, (unsigned)blockIdx.x + 1u);
      atomicExch(p.status + 2, (unsigned)(k + m * NP));
      const int64_t issued = m + L < n ? m + L : n;
      for (int64_t q = m; q < issued; ++q) {
        if (!mbar_wait_bounded(bar0 + 8u * (uint32_t)(q % S), (uint32_t)((q / S) & 1))) {
          atomicOr(p.status, kStatusDrainTimeout);
          break;
        }
      }
      bulk_wait_all();
      return;
    }
#if UA2A_STORE_FENCE
    fence_proxy_async_smem();
#endif
    issue_store(m);
    const int64_t next = m + L;
    if (next < n) {
      bulk_wait_read_n(S - L);  // the store of tile next - S has read its stage
      issue_load(next);
    }
  }
  bulk_wait_all();
}

// Self-test of the failure path: one thread initialises an mbarrier that
// nothing ever arrives on, waits for it through mbar_wait_bounded with a short
// limit, and records the expiry in the status words exactly as the copy
// kernel does. No memory other than the status words is touched.
// (A template, like the copy kernels, so that it is instantiated only in the
// translation unit that launches it.)
template <int kUnused = 0>
__global__ void __launch_bounds__(32, 1)
    ua2a_wait_selftest_kernel(unsigned int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_addr(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  if (!mbar_wait_bounded(b, 0, limit_ns)) {
    atomicOr(status, kStatusWaitTimeout);
    atomicExch(status + 1, (unsigned)blockIdx.x + 1u);
    atomicExch(status + 2, 0u);
  }
}

}  // namespace ua2a
