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
// One thread per CTA drives a ring of `stages` shared-memory tiles over the
// units this CTA owns (u = blockIdx.x + i*gridDim.x, a static round-robin
// persistent schedule). Every mbarrier wait is bounded in time; on expiry the
// kernel records the failure in the context's status word, waits (bounded)
// for its own copies still in flight and returns.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "ulysses_a2a.h"

namespace ua2a {

constexpr int kTmaStagesMax = 16;
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
  int32_t tiles_per_block;                      // T = ceil(S_local / S_tile)
  int32_t b0;                                   // first plane of this launch
  int32_t nb;                                   // planes in this launch
  uint32_t tile_bytes;                          // full box bytes (clipped rows included)
  uint32_t stage_bytes;                         // tile_bytes rounded up to 1 KB
  int32_t stages;
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
// kWaitLimitNs (checked every 256 polls) and at most 2^30 polls.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && global_ns() - t0 > kWaitLimitNs) return false;
  }
  return false;
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(c4)
      : "memory");
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group"
      " [%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_store_5d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group"
      " [%0, {%2, %3, %4, %5, %6}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// All but the newest N bulk groups have finished READING shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

struct UnitCoord {
  int r, b, j, s0;
};

__device__ __forceinline__ UnitCoord decode_unit(const TmaParams& p, int64_t u) {
  // u = ((r * nb + b_rel) * w + j) * T + t
  UnitCoord c;
  const int64_t t = u % p.tiles_per_block;
  int64_t q = u / p.tiles_per_block;
  c.j = (int)(q % p.w);
  q /= p.w;
  c.b = p.b0 + (int)(q % p.nb);
  c.r = (int)(q / p.nb);
  c.s0 = (int)(t * p.rows_per_tile);
  return c;
}

template <int MODE>
__global__ void __launch_bounds__(32, 1) ua2a_tma_kernel(const __grid_constant__ TmaParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[kTmaStagesMax];
  if (threadIdx.x != 0) return;

  const int64_t G = gridDim.x;
  const int64_t first = blockIdx.x;
  if (first >= p.units) return;
  const int64_t n = (p.units - first + G - 1) / G;  // units owned by this CTA
  const int S = p.stages;
  const uint32_t smem0 = smem_addr(smem);
  const uint32_t bar0 = smem_addr(full);

  for (int s = 0; s < S; ++s) mbar_init(bar0 + 8u * s, 1);
  fence_barrier_init();
  fence_proxy_async_smem();

  auto issue_load = [&](int64_t i) {
    const int s = (int)(i % S);
    const UnitCoord c = decode_unit(p, first + i * G);
    const uint32_t bar = bar0 + 8u * s;
    const uint32_t dst = smem0 + (uint32_t)s * p.stage_bytes;
    mbar_arrive_expect_tx(bar, p.tile_bytes);
    if (MODE == 0)
      tma_load_4d(dst, &p.strided[c.j], bar, 0, c.r * p.Hw, c.s0, c.b);
    else
      tma_load_5d(dst, &p.gathered[c.r], bar, 0, 0, c.s0, c.j, c.b);
  };
  auto issue_store = [&](int64_t i) {
    const int s = (int)(i % S);
    const UnitCoord c = decode_unit(p, first + i * G);
    const uint32_t src = smem0 + (uint32_t)s * p.stage_bytes;
    if (MODE == 0)
      tma_store_5d(&p.gathered[c.r], src, 0, 0, c.s0, c.j, c.b);
    else
      tma_store_4d(&p.strided[c.j], src, 0, c.r * p.Hw, c.s0, c.b);
    bulk_commit();
  };

  const int64_t pre = n < S ? n : S;
  for (int64_t i = 0; i < pre; ++i) issue_load(i);

  for (int64_t i = 0; i < n; ++i) {
    const int s = (int)(i % S);
    const uint32_t parity = (uint32_t)((i / S) & 1);
    if (!mbar_wait_bounded(bar0 + 8u * s, parity)) {
      // Record, then drain: loads i .. issued-1 may still be landing in this
      // CTA's shared memory; wait for each once more (bounded) before leaving.
      atomicOr(p.status, kStatusWaitTimeout);
      atomicExch(p.status + 1, (unsigned)blockIdx.x + 1u);
      atomicExch(p.status + 2, (unsigned)i);
      const int64_t issued = (i >= 1 ? (i - 1 + S < n ? i - 1 + S : n) : pre);
      for (int64_t k = i; k < issued; ++k) {
        if (!mbar_wait_bounded(bar0 + 8u * (uint32_t)(k % S), (uint32_t)((k / S) & 1))) {
          atomicOr(p.status, kStatusDrainTimeout);
          break;
        }
      }
      bulk_wait_all();
      return;
    }
    fence_proxy_async_smem();
    issue_store(i);
    // Refill the stage that held tile i-1 once its store has read it out.
    if (i >= 1 && i - 1 + S < n) {
      bulk_wait_read<1>();
      issue_load(i - 1 + S);
    }
  }
  bulk_wait_all();
}

}  // namespace ua2a
