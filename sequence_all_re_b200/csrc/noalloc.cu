// noalloc.cu - the allocation-free entry point of the Ulysses 4D all-to-all
// re-layout (ulysses_a2a_run_noalloc in include/ulysses_a2a.h).
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "internal.h"

using namespace ua2a;
using ua2a::StageParams;
using ua2a::TmaParams;
using ua2a::VecParams;

// ---------------------------------------------------------------------------
// Allocation-free entry point (ulysses_a2a_run_noalloc).
//
// For callers that may not allocate device memory themselves: a process whose
// device memory is owned by another allocator under a fixed budget, or a host
// thread running where a cudaMalloc/cudaFree (which can synchronise the device)
// is not allowed. ulysses_a2a_create allocates the TMA kernel's status records;
// this entry point runs the same kernels with those records in a file-scope
// static device array instead, and needs no context.
//
// The array is modest and fixed: kNoAllocSlots records of 16 bytes (1 KiB),
// one record per TMA kernel launch of a call (a chunked call launches once per
// plane; the VEC kernel has no bounded wait and uses none), held by every GPU
// that loads this library until the process exits.
// Every call shares it and it keeps the last call's contents: each call clears
// the records it uses, on its stream, before launching, so two calls whose work
// overlaps on the GPU (different streams, or different host threads) race on it.
// ---------------------------------------------------------------------------

namespace {
constexpr int kNoAllocSlots = 64;
constexpr int kNoAllocSlotWords = 4;
constexpr int kNoAllocMaxDevices = 64;
}  // namespace

static __device__ __align__(256) unsigned int ua2a_noalloc_scratch[kNoAllocSlots * kNoAllocSlotWords];

namespace {

struct NoAllocDevice {
  std::mutex mu;
  bool ready = false;               // set-up done and succeeded on this device
  unsigned int* scratch = nullptr;  // this device's address of ua2a_noalloc_scratch
  int num_sms = 0;
};

NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];
std::once_flag g_noalloc_driver_once;
PFN_cuTensorMapEncodeTiled_v12000 g_noalloc_encode = nullptr;
PFN_cuMemGetAddressRange_v3020 g_noalloc_range = nullptr;

int noalloc_report(char* err, size_t errlen, int rc, const char* fmt, long long a = 0,
                   long long b = 0) {
  if (err && errlen) std::snprintf(err, errlen, fmt, a, b);
  return rc;
}

// Per device, with that device current: resolve the array's device address
// (the symbol itself is only a host-side stand-in) and set the kernels' shared
// memory limit. Only a successful set-up is remembered; after a failure (for
// example a cudaFuncSetAttribute refused during a stream capture) the next
// call on that device tries again.
int noalloc_setup(NoAllocDevice& st, int dev, char* err, size_t errlen) {
  std::lock_guard<std::mutex> lock(st.mu);
  if (st.ready) return ULYSSES_A2A_OK;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major < 10) {
    cudaGetLastError();
    return noalloc_report(err, errlen, ULYSSES_A2A_ERR_DEVICE, "device %lld is not an sm_100 GPU",
                          dev);
  }
  void* addr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&addr, ua2a_noalloc_scratch);
  if (e != cudaSuccess || addr == nullptr) {
    cudaGetLastError();
    if (err && errlen)
      std::snprintf(err, errlen, "cudaGetSymbolAddress failed: %s", cudaGetErrorName(e));
    return ULYSSES_A2A_ERR_CUDA;
  }
  if (tma_allow_max_smem() != cudaSuccess || stage_allow_max_smem() != cudaSuccess) {
    cudaGetLastError();
    return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA,
                          "cudaFuncSetAttribute failed (set-up is retried on the next call)");
  }
  st.num_sms = prop.multiProcessorCount;
  st.scratch = static_cast<unsigned int*>(addr);
  st.ready = true;
  return ULYSSES_A2A_OK;
}

bool noalloc_encode(CUtensorMap* m, int rank, const void* base, const cuuint64_t* dims,
                    const cuuint64_t* strides, const cuuint32_t* box, int E) {
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return g_noalloc_encode(m, map_dtype(E), (cuuint32_t)rank, const_cast<void*>(base), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          UA2A_L2_PROMOTION,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

static int ua2a_impl_run_noalloc(const void* const* in_slabs, void* const* out_slabs,
                                       int64_t B, int64_t S_local, int64_t H, int64_t D, int w,
                                       int mode, int chunked, int elem_bytes, void* stream,
                                       int wait, char* err, size_t errlen) {
  if (err && errlen) err[0] = '\0';
  std::call_once(g_noalloc_driver_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_noalloc_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_noalloc_range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
    cudaGetLastError();
  });
  if (g_noalloc_encode == nullptr)
    return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (chunked == ULYSSES_A2A_CHUNKED_WINDOW)
    return noalloc_report(err, errlen, ULYSSES_A2A_ERR_UNSUPPORTED,
                          "chunked = 2 needs a staging window; use chunked 0 or 1 here");

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) {
    cudaGetLastError();
    return noalloc_report(err, errlen, ULYSSES_A2A_ERR_DEVICE, "no usable current CUDA device");
  }
  NoAllocDevice& st = g_noalloc_dev[dev];
  const int setup_rc = noalloc_setup(st, dev, err, errlen);
  if (setup_rc != ULYSSES_A2A_OK) return setup_rc;

  // the same checks as ulysses_a2a_run, before anything is launched
  ulysses_a2a_plan_t pl;
  int rc = ua2a::make_plan(in_slabs, out_slabs, B, S_local, H, D, w, mode, chunked, elem_bytes,
                           ULYSSES_A2A_PATH_AUTO, ua2a::Tuning{}, st.num_sms, &pl, nullptr);
  if (rc != ULYSSES_A2A_OK) {
    std::string msg;
    ua2a::make_plan(in_slabs, out_slabs, B, S_local, H, D, w, mode, chunked, elem_bytes,
                    ULYSSES_A2A_PATH_AUTO, ua2a::Tuning{}, st.num_sms, &pl, &msg);
    if (err && errlen) std::snprintf(err, errlen, "%s", msg.c_str());
    return rc;
  }
  if (pl.units == 0) return ULYSSES_A2A_OK;  // empty: nothing to do
  // Only the TMA kernel writes status records (one per launch); the VEC kernel
  // has no bounded wait and needs none.
  const bool tma = pl.path == ULYSSES_A2A_PATH_TMA;
  const int slots = tma ? pl.launches : 0;
  if (slots > kNoAllocSlots)
    return noalloc_report(err, errlen, ULYSSES_A2A_ERR_UNSUPPORTED,
                          "chunked call over %lld planes needs %lld status records; the static "
                          "scratch holds 64 (1 KiB): split the call or use ulysses_a2a_run",
                          (long long)slots, (long long)slots);
  const int64_t slab_bytes = pl.payload_bytes / w;
  for (int side = 0; side < 2; ++side) {
    for (int k = 0; k < w; ++k) {
      const void* p = side == 0 ? in_slabs[k] : out_slabs[k];
      cudaPointerAttributes a;
      if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        if (err && errlen)
          std::snprintf(err, errlen, "%s slab %d is not a CUDA pointer", side ? "output" : "input", k);
        return ULYSSES_A2A_ERR_DEVICE;
      }
      if (!(a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) || a.device != dev) {
        if (err && errlen)
          std::snprintf(err, errlen, "%s slab %d is not device memory of the current device %d",
                        side ? "output" : "input", k, dev);
        return ULYSSES_A2A_ERR_DEVICE;
      }
      if (g_noalloc_range && a.type == cudaMemoryTypeDevice) {
        CUdeviceptr base = 0;
        size_t size = 0;
        if (g_noalloc_range(&base, &size, (CUdeviceptr)(uintptr_t)p) == CUDA_SUCCESS &&
            (uintptr_t)p + (uintptr_t)slab_bytes > (uintptr_t)base + size) {
          if (err && errlen)
            std::snprintf(err, errlen, "%s slab %d runs past the end of its allocation",
                          side ? "output" : "input", k);
          return ULYSSES_A2A_ERR_DEVICE;
        }
      }
    }
  }

  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (slots > 0) {
    // the records of this call start at zero (the array keeps the previous call's)
    e = cudaMemsetAsync(st.scratch, 0, sizeof(unsigned int) * kNoAllocSlotWords * slots, st_);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA,
                            "cudaMemsetAsync of the status records failed");
    }
  }
  const int64_t nb = chunked ? 1 : B;
  if (tma) {
    TmaParams p;
    std::memset(&p, 0, sizeof(p));
    const int64_t E = elem_bytes, Hw = H / w, rows = pl.rows_per_tile;
    for (int k = 0; k < w; ++k) {
      const void* strided = mode == 0 ? in_slabs[k] : out_slabs[k];
      const void* gathered = mode == 0 ? out_slabs[k] : in_slabs[k];
      const cuuint64_t sd[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S_local, (cuuint64_t)B};
      const cuuint64_t ss[3] = {(cuuint64_t)(D * E), (cuuint64_t)(H * D * E),
                                (cuuint64_t)(S_local * H * D * E)};
      const cuuint32_t sb[4] = {(cuuint32_t)D, (cuuint32_t)Hw, (cuuint32_t)rows, 1};
      const cuuint64_t gd[5] = {(cuuint64_t)D, (cuuint64_t)Hw, (cuuint64_t)S_local, (cuuint64_t)w,
                                (cuuint64_t)B};
      const cuuint64_t gs[4] = {(cuuint64_t)(D * E), (cuuint64_t)(Hw * D * E),
                                (cuuint64_t)(S_local * Hw * D * E),
                                (cuuint64_t)(w * S_local * Hw * D * E)};
      const cuuint32_t gb[5] = {(cuuint32_t)D, (cuuint32_t)Hw, (cuuint32_t)rows, 1, 1};
      if (!noalloc_encode(&p.strided[k], 4, strided, sd, ss, sb, elem_bytes) ||
          !noalloc_encode(&p.gathered[k], 5, gathered, gd, gs, gb, elem_bytes))
        return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA, "cuTensorMapEncodeTiled failed for slab %lld", k);
    }
    p.units = pl.units;
    p.w = w;
    p.Hw = (int32_t)Hw;
    p.rows_per_tile = (int32_t)rows;
    p.tiles_per_block = (int32_t)pl.tiles_per_block;
    p.tile0 = 0;
    p.nb = (int32_t)nb;
    p.tile_bytes = (uint32_t)(rows * pl.row_bytes);
    p.stage_bytes = (p.tile_bytes + 1023u) / 1024u * 1024u;
    p.stages = pl.stages / pl.producers;
    p.lookahead = pl.lookahead;
    p.producers = pl.producers;
    p.order = pl.order;
    p.chunk_units = pl.chunk_units;
    for (int l = 0; l < pl.launches; ++l) {
      p.b0 = chunked ? l : 0;
      p.status = st.scratch + kNoAllocSlotWords * l;
      e = launch_tma(mode, pl.grid, pl.block, (size_t)pl.smem_bytes, st_, p);
      if (e != cudaSuccess)
        return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA, "TMA kernel launch failed (plane %lld)", l);
    }
  } else if (pl.path == ULYSSES_A2A_PATH_STAGED) {
    StageParams p = stage_params(S_local, w, 1, elem_bytes, pl, pl.tiles_per_block, pl.units);
    for (int k = 0; k < w; ++k) {
      p.in[k] = static_cast<const char*>(in_slabs[k]);
      p.out[k] = static_cast<char*>(out_slabs[k]);
    }
    for (int l = 0; l < pl.launches; ++l) {
      p.b0 = chunked ? l : 0;
      e = launch_stage(p, pl.vec_bytes, pl.fixed_phase, mode, pl.grid, pl.block,
                       (size_t)pl.smem_bytes, st_);
      if (e != cudaSuccess)
        return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA, "staged kernel launch failed (plane %lld)", l);
    }
  } else {
    VecParams p = vec_params(in_slabs, out_slabs, w, w, S_local, w, elem_bytes, pl, pl.units, nb,
                             pl.tiles_per_block, w, w, 0u, 1u, 0u, 0);
    for (int l = 0; l < pl.launches; ++l) {
      p.b0 = chunked ? l : 0;
      e = launch_vec(p, pl.vec_bytes, pl.peeled, mode, pl.grid, pl.block, st_);
      if (e != cudaSuccess)
        return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA, "VEC kernel launch failed (plane %lld)", l);
    }
  }
  if (!wait) return ULYSSES_A2A_OK;
  e = cudaStreamSynchronize(st_);
  if (e != cudaSuccess)
    return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA, "cudaStreamSynchronize failed");
  if (slots == 0) return ULYSSES_A2A_OK;
  unsigned int h[kNoAllocSlots * kNoAllocSlotWords];
  e = cudaMemcpy(h, st.scratch, sizeof(unsigned int) * kNoAllocSlotWords * slots, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess)
    return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA, "reading the status records failed");
  for (int l = 0; l < slots; ++l) {
    if (h[kNoAllocSlotWords * l] != 0)
      return noalloc_report(err, errlen, ULYSSES_A2A_ERR_TIMEOUT,
                            "a TMA wait gave up in launch %lld (flags 0x%llx)", l,
                            h[kNoAllocSlotWords * l]);
  }
  return ULYSSES_A2A_OK;
}

extern "C" {

int ulysses_a2a_run_noalloc(const void* const* in_slabs, void* const* out_slabs, int64_t B,
                            int64_t S_local, int64_t H, int64_t D, int w, int mode, int chunked,
                            int elem_bytes, void* stream, int wait, char* err, size_t errlen) {
  return no_throw([&] { return ua2a_impl_run_noalloc(in_slabs, out_slabs, B, S_local, H, D, w, mode,
                                                     chunked, elem_bytes, stream, wait, err,
                                                     errlen); });
}

}  // extern "C"
