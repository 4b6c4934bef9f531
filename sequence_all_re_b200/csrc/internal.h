// internal.h - declarations shared by the library's translation units:
//   ulysses_a2a.cu  the context, the single-GPU entry points and every kernel
//                   launch (the kernels are instantiated there only);
//   peer.cu         the multi-GPU exchange through published windows;
//   noalloc.cu      the allocation-free entry point.
// Not part of the public ABI (include/ulysses_a2a.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <new>
#include <string>
#include <vector>

#include "kernels_peel.cuh"
#include "kernels_phase.cuh"
#include "kernels_stage.cuh"
#include "kernels_tma.cuh"
#include "kernels_vec.cuh"
#include "plan.h"
#include "ulysses_a2a.h"

// L2 fetch granularity the TMA unit uses for the tensor maps (tunable at build time).
#ifndef UA2A_L2_PROMOTION
#define UA2A_L2_PROMOTION CU_TENSOR_MAP_L2_PROMOTION_L2_256B
#endif

namespace ua2a {

constexpr int kTmaCacheEntries = 16;


struct TmaCacheEntry {
  bool valid = false;
  uint64_t stamp = 0;
  int mode = 0, w = 0;
  int64_t B = 0, S = 0, H = 0, D = 0, rows = 0, pitch = 0;
  const void* in[ULYSSES_A2A_MAX_W_TMA] = {};
  void* out[ULYSSES_A2A_MAX_W_TMA] = {};
  TmaParams params;  // tensor maps + geometry (b0/nb/status filled per launch)
};

}  // namespace ua2a


struct ulysses_a2a_ctx {
  int device = 0;
  int elem_bytes = 2;
  int num_sms = 148;
  int forced_path = ULYSSES_A2A_PATH_AUTO;
  ua2a::Tuning tuning;
  unsigned int* d_status = nullptr;  // 4 words, see kernels_tma.cuh
  std::string last_error;
  uint64_t launches = 0;
  uint64_t stamp = 0;
  ua2a::TmaCacheEntry tma_cache[ua2a::kTmaCacheEntries];
  bool tma_smem_set[2] = {false, false};
  bool stage_smem_set = false;
  int64_t tma_smem_set_bytes[2] = {0, 0};
  // run_host staging: one device buffer carved into 2w slabs
  void* d_stage = nullptr;
  size_t stage_bytes = 0;
  cudaStream_t copy_stream[2] = {nullptr, nullptr};  // H2D, D2H
  // chunked = 2: the staging window (one plane of every input slab)
  void* d_window = nullptr;
  size_t window_bytes = 0;
  std::vector<cudaEvent_t> copy_events;              // start + 2 per chunk
  PFN_cuTensorMapEncodeTiled_v12000 encode_tiled = nullptr;
  PFN_cuMemGetAddressRange_v3020 get_range = nullptr;
};

namespace ua2a {

// Switch to the context's device for the lifetime of the guard.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    ok = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

// Record msg as ctx's last error and return code.
int fail(ulysses_a2a_ctx* ctx, int code, const std::string& msg);
// ULYSSES_A2A_ERR_CUDA with the name and text of a CUDA error.
int cuda_fail(ulysses_a2a_ctx* ctx, const char* what, cudaError_t e);
// Tensor-map element type for elem_bytes.
CUtensorMapDataType map_dtype(int E);
// Every one of the w slabs is device memory of ctx's device and lies inside
// the allocation that contains its start.
int check_residency(ulysses_a2a_ctx* ctx, const void* const* ptrs, int w, int64_t bytes,
                    const char* what);
// Kernel launches (programmatic stream serialization).
cudaError_t launch_tma(int mode, int grid, int block, size_t smem, cudaStream_t st,
                       const TmaParams& p);
cudaError_t launch_vec(const VecParams& p, int vec_bytes, int peeled, int mode, int grid,
                       int block, cudaStream_t st);
// VEC-path kernel parameters for a plan (b0 left for the caller): nr head
// groups from r0 in steps of r_stride, nj sequence blocks from j0, nb planes
// and nt tiles of each (r, b, j) block from tile0, `units` units in all.
VecParams vec_params(const void* const* in, void* const* out, int nin, int nout, int64_t S, int w,
                     int E, const ulysses_a2a_plan_t& pl, int64_t units, int64_t nb, int64_t nt,
                     int nr, int nj, uint32_t r0, uint32_t r_stride, uint32_t j0, int64_t tile0);
// One staged launch: the fixed-phase kernel when fixed_phase is set (pieces
// of 8 bytes or less), else the per-piece kernel.
cudaError_t launch_stage(const StageParams& p, int piece_bytes, int fixed_phase, int mode, int grid,
                         int block, size_t smem, cudaStream_t st);
// Let every staged kernel (both forms) use up to kStageSmemMax of dynamic
// shared memory.
cudaError_t stage_allow_max_smem();
// Staged-kernel parameters for a plan (slab pointers, tile0 and b0 left for
// the caller): nt tiles per (b, j) block, `units` units in the launch.
StageParams stage_params(int64_t S, int w, int ntensors, int E, const ulysses_a2a_plan_t& pl,
                         int64_t nt, int64_t units);
// Let both TMA kernels use up to kTmaSmemMax of dynamic shared memory (on the
// current device; the attribute belongs to the instantiations launched above).
cudaError_t tma_allow_max_smem();
// Launch the planned kernel(s) for tiles [tile0, tile0 + ntiles) of every
// (r, b, j) block (ntiles < 0: the whole block). only_out >= 0 (VEC path
// only) restricts the launch to the blocks of output slab only_out: r fixed in
// mode 0, j fixed in mode 1. ntensors > 1 (VEC path only): head-packed
// tensors, r ranging over ntensors*w head groups.
int run_device(ulysses_a2a_ctx* ctx, const void* const* in, void* const* out, int64_t B, int64_t S,
               int64_t H, int64_t D, int w, int mode, int chunked, cudaStream_t st,
               const ulysses_a2a_plan_t& pl, int64_t tile0 = 0, int64_t ntiles = -1,
               int only_out = -1, int ntensors = 1);
// make_plan with ctx's element size, forced path, tuning and SM count.
int plan_for(ulysses_a2a_ctx* ctx, const void* const* in, void* const* out, int64_t B, int64_t S,
             int64_t H, int64_t D, int w, int mode, int chunked, ulysses_a2a_plan_t* pl,
             int64_t row_pitch = 0, int ntensors = 1);

// The exported entry points: no exception may cross the C ABI. A failed host
// allocation inside the library becomes ULYSSES_A2A_ERR_NOMEM, any other
// exception ULYSSES_A2A_ERR_INTERNAL.
template <typename F>
int no_throw(F&& f) noexcept {
  try {
    return f();
  } catch (const std::bad_alloc&) {
    return ULYSSES_A2A_ERR_NOMEM;
  } catch (...) {
    return ULYSSES_A2A_ERR_INTERNAL;
  }
}

}  // namespace ua2a
