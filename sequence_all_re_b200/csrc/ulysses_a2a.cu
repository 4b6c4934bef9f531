// ulysses_a2a.cu - C ABI of the B200 Ulysses 4D all-to-all re-layout.
//
// Implements include/ulysses_a2a.h. The operation and its argument convention
// follow the FastVideo API docs, fastvideo.distributed.device_communicators
// .ulysses_a2a, `run_armed`: the native op always receives the mode-0-local
// tuple (B, S_local, H, D); mode 0 produces [B, S_local*w, H/w, D] per rank,
// mode 1 produces [B, S_local, H, D]; the chunked variant runs the op once per
// plane on one-plane views, each plane finishing (stream order) before the
// next starts.
//
// On one GPU every rank slab is local, so the all-to-all is a permutation and
// the work is pure data movement: two kernels (kernels_tma.cuh,
// kernels_vec.cuh), picked per shape by the host planner (plan.h). The context
// plays the part of the page's reusable communication handle: it holds the
// rank-slab descriptor table (TMA tensor maps, cached per pointer set and
// shape), the device status word of the bounded waits, and the device staging
// buffers of the host-buffer entry point (grown on demand, like the page's
// window `_build`/grow).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <chrono>
#include <cstring>
#include <functional>
#include <mutex>
#include <new>
#include <random>
#include <string>
#include <vector>

#include <unistd.h>

#include "kernels_tma.cuh"
#include "kernels_vec.cuh"
#include "plan.h"
#include "ulysses_a2a.h"

// L2 fetch granularity the TMA unit uses for the tensor maps (tunable at build time).
#ifndef UA2A_L2_PROMOTION
#define UA2A_L2_PROMOTION CU_TENSOR_MAP_L2_PROMOTION_L2_256B
#endif

using ua2a::TmaParams;
using ua2a::VecParams;

static_assert(ua2a::kVecResidentCtasPerSm == ua2a::kVecMinBlocksPerSm,
              "the planner's VEC residency must match the kernel's launch bound");

namespace {

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

}  // namespace

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
  TmaCacheEntry tma_cache[kTmaCacheEntries];
  bool tma_smem_set[2] = {false, false};
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

namespace {

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

int fail(ulysses_a2a_ctx* ctx, int code, const std::string& msg) {
  if (ctx) ctx->last_error = msg;
  return code;
}

int cuda_fail(ulysses_a2a_ctx* ctx, const char* what, cudaError_t e) {
  return fail(ctx, ULYSSES_A2A_ERR_CUDA,
              std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")");
}

CUtensorMapDataType map_dtype(int E) {
  switch (E) {
    case 1: return CU_TENSOR_MAP_DATA_TYPE_UINT8;
    case 2: return CU_TENSOR_MAP_DATA_TYPE_UINT16;
    case 4: return CU_TENSOR_MAP_DATA_TYPE_UINT32;
    default: return CU_TENSOR_MAP_DATA_TYPE_UINT64;
  }
}

// Tensor maps of one strided-side slab [B, S, H, D] and one gathered-side slab
// [B, S*w, H/w, D] (viewed as [B, w, S, H/w, D] so rows stop at S per block).
int encode_strided(ulysses_a2a_ctx* ctx, CUtensorMap* m, const void* base, int64_t B, int64_t S,
                   int64_t H, int64_t D, int64_t Hw, int64_t rows, int64_t pitch) {
  const int64_t E = ctx->elem_bytes;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)(D * E), (cuuint64_t)(pitch * E), (cuuint64_t)(S * pitch * E)};
  cuuint32_t box[4] = {(cuuint32_t)D, (cuuint32_t)Hw, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = ctx->encode_tiled(m, map_dtype((int)E), 4, const_cast<void*>(base), dims, strides, box,
                                 estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                 UA2A_L2_PROMOTION, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(ctx, ULYSSES_A2A_ERR_CUDA, "cuTensorMapEncodeTiled (strided side) failed: " + std::to_string((int)r));
  return ULYSSES_A2A_OK;
}

int encode_gathered(ulysses_a2a_ctx* ctx, CUtensorMap* m, const void* base, int64_t B, int64_t S,
                    int64_t Hw, int64_t D, int w, int64_t rows) {
  const int64_t E = ctx->elem_bytes;
  cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)Hw, (cuuint64_t)S, (cuuint64_t)w, (cuuint64_t)B};
  cuuint64_t strides[4] = {(cuuint64_t)(D * E), (cuuint64_t)(Hw * D * E), (cuuint64_t)(S * Hw * D * E),
                           (cuuint64_t)(w * S * Hw * D * E)};
  cuuint32_t box[5] = {(cuuint32_t)D, (cuuint32_t)Hw, (cuuint32_t)rows, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = ctx->encode_tiled(m, map_dtype((int)E), 5, const_cast<void*>(base), dims, strides, box,
                                 estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                 UA2A_L2_PROMOTION, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(ctx, ULYSSES_A2A_ERR_CUDA, "cuTensorMapEncodeTiled (gathered side) failed: " + std::to_string((int)r));
  return ULYSSES_A2A_OK;
}

// Find or build the descriptor table for this pointer set and shape.
int tma_params_for(ulysses_a2a_ctx* ctx, const void* const* in, void* const* out, int64_t B,
                   int64_t S, int64_t H, int64_t D, int w, int mode, const ulysses_a2a_plan_t& pl,
                   TmaParams** result) {
  const int64_t rows = pl.rows_per_tile;
  const int64_t pitch = pl.row_pitch;
  TmaCacheEntry* victim = &ctx->tma_cache[0];
  for (auto& e : ctx->tma_cache) {
    if (e.valid && e.mode == mode && e.w == w && e.B == B && e.S == S && e.H == H && e.D == D &&
        e.rows == rows && e.pitch == pitch) {
      bool same = true;
      for (int k = 0; k < w && same; ++k) same = e.in[k] == in[k] && e.out[k] == out[k];
      if (same) {
        e.stamp = ++ctx->stamp;
        e.params.stages = pl.stages / pl.producers;
        e.params.lookahead = pl.lookahead;
        e.params.producers = pl.producers;
        e.params.order = pl.order;
        e.params.chunk_units = pl.chunk_units;
        *result = &e.params;
        return ULYSSES_A2A_OK;
      }
    }
    if (!e.valid || e.stamp < victim->stamp) victim = &e;
  }
  TmaCacheEntry fresh;
  const int64_t Hw = H / w;
  // mode 0 reads the strided side (inputs) and writes the gathered side (outputs);
  // mode 1 the reverse
  for (int k = 0; k < w; ++k) {
    const void* strided = mode == 0 ? in[k] : out[k];
    const void* gathered = mode == 0 ? out[k] : in[k];
    int rc = encode_strided(ctx, &fresh.params.strided[k], strided, B, S, H, D, Hw, rows, pitch);
    if (rc) return rc;
    rc = encode_gathered(ctx, &fresh.params.gathered[k], gathered, B, S, Hw, D, w, rows);
    if (rc) return rc;
    fresh.in[k] = in[k];
    fresh.out[k] = out[k];
  }
  fresh.valid = true;
  fresh.stamp = ++ctx->stamp;
  fresh.mode = mode;
  fresh.w = w;
  fresh.B = B;
  fresh.S = S;
  fresh.H = H;
  fresh.D = D;
  fresh.rows = rows;
  fresh.pitch = pitch;
  TmaParams& p = fresh.params;
  p.status = ctx->d_status;
  p.w = w;
  p.Hw = (int32_t)Hw;
  p.rows_per_tile = (int32_t)rows;
  p.tiles_per_block = (int32_t)pl.tiles_per_block;
  p.tile_bytes = (uint32_t)(rows * pl.row_bytes);
  p.stage_bytes = (uint32_t)((p.tile_bytes + 1023u) / 1024u * 1024u);
  p.stages = pl.stages / pl.producers;
  p.lookahead = pl.lookahead;
  p.producers = pl.producers;
  p.order = pl.order;
  p.chunk_units = pl.chunk_units;
  *victim = fresh;
  *result = &victim->params;
  return ULYSSES_A2A_OK;
}

// Every slab must sit in device memory of ctx's device, inside one allocation.
int check_residency(ulysses_a2a_ctx* ctx, const void* const* ptrs, int w, int64_t bytes,
                    const char* what) {
  for (int k = 0; k < w; ++k) {
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, ptrs[k]);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(ctx, ULYSSES_A2A_ERR_DEVICE, std::string(what) + " slab " + std::to_string(k) +
                                                   ": not a CUDA pointer");
    }
    if (!(a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) || a.device != ctx->device)
      return fail(ctx, ULYSSES_A2A_ERR_DEVICE, std::string(what) + " slab " + std::to_string(k) +
                                                   " is not device memory of device " +
                                                   std::to_string(ctx->device));
    if (ctx->get_range && a.type == cudaMemoryTypeDevice) {
      CUdeviceptr base = 0;
      size_t size = 0;
      if (ctx->get_range(&base, &size, (CUdeviceptr)(uintptr_t)ptrs[k]) == CUDA_SUCCESS) {
        const uintptr_t p = (uintptr_t)ptrs[k];
        if (p + (uintptr_t)bytes > (uintptr_t)base + size)
          return fail(ctx, ULYSSES_A2A_ERR_DEVICE, std::string(what) + " slab " + std::to_string(k) +
                                                       " runs past the end of its allocation");
      }
    }
  }
  return ULYSSES_A2A_OK;
}

// Launch with programmatic stream serialization (the kernels start with
// griddepcontrol.wait, so a dependent launch cannot overtake its producer).
template <typename Kernel, typename Params>
cudaError_t launch_pdl(Kernel kernel, int grid, int block, size_t smem, cudaStream_t st,
                       const Params& p) {
#if UA2A_PDL
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, p);
  if (e != cudaSuccess) return e;
#else
  kernel<<<grid, block, smem, st>>>(p);
#endif
  return cudaGetLastError();
}

cudaError_t launch_tma(int mode, int grid, int block, size_t smem, cudaStream_t st,
                       const TmaParams& p) {
  return mode == 0 ? launch_pdl(ua2a::ua2a_tma_kernel<0>, grid, block, smem, st, p)
                   : launch_pdl(ua2a::ua2a_tma_kernel<1>, grid, block, smem, st, p);
}

template <typename V>
cudaError_t launch_vec_t(const VecParams& p, int mode, int grid, int block, cudaStream_t st) {
  return mode == 0 ? launch_pdl(ua2a::ua2a_vec_kernel<V, 0, 4>, grid, block, 0, st, p)
                   : launch_pdl(ua2a::ua2a_vec_kernel<V, 1, 4>, grid, block, 0, st, p);
}

cudaError_t launch_vec(const VecParams& p, int vec_bytes, int mode, int grid, int block,
                       cudaStream_t st) {
  switch (vec_bytes) {
    case 16: return launch_vec_t<uint4>(p, mode, grid, block, st);
    case 8: return launch_vec_t<uint2>(p, mode, grid, block, st);
    case 4: return launch_vec_t<unsigned int>(p, mode, grid, block, st);
    case 2: return launch_vec_t<unsigned short>(p, mode, grid, block, st);
    default: return launch_vec_t<unsigned char>(p, mode, grid, block, st);
  }
}

// Launch the planned kernel(s) for tiles [tile0, tile0 + ntiles) of every
// (r, b, j) block (ntiles < 0: the whole block). only_out >= 0 (VEC path
// only) restricts the launch to the blocks of output slab only_out: r fixed in
// mode 0, j fixed in mode 1. ntensors > 1 (VEC path only): head-packed
// tensors, r ranging over ntensors*w head groups.
int run_device(ulysses_a2a_ctx* ctx, const void* const* in, void* const* out, int64_t B, int64_t S,
               int64_t H, int64_t D, int w, int mode, int chunked, cudaStream_t st,
               const ulysses_a2a_plan_t& pl, int64_t tile0 = 0, int64_t ntiles = -1,
               int only_out = -1, int ntensors = 1) {
  const int64_t nb = chunked ? 1 : B;
  const int launches = chunked ? (int)B : 1;
  const int64_t nt = ntiles < 0 ? pl.tiles_per_block : ntiles;
  const int nr = (only_out >= 0 && mode == 0) ? 1 : w * ntensors;
  const int nj = (only_out >= 0 && mode == 1) ? 1 : w;
  const int64_t units = (int64_t)nr * nb * nj * nt;
  if ((only_out >= 0 || ntensors > 1) && pl.path != ULYSSES_A2A_PATH_VEC)
    return fail(ctx, ULYSSES_A2A_ERR_UNSUPPORTED, "one-output and packed launches use the VEC path");
  int grid = pl.grid;
  if (nt != pl.tiles_per_block) {
    if (pl.path == ULYSSES_A2A_PATH_TMA && pl.chunk_units > 0)
      grid = (int)((units + pl.chunk_units - 1) / pl.chunk_units);
    else if (units < grid)
      grid = (int)units;
  }
  if (pl.path == ULYSSES_A2A_PATH_TMA) {
    TmaParams* cached = nullptr;
    int rc = tma_params_for(ctx, in, out, B, S, H, D, w, mode, pl, &cached);
    if (rc) return rc;
    TmaParams p = *cached;
    p.status = ctx->d_status;
    p.nb = (int32_t)nb;
    p.units = units;
    p.tiles_per_block = (int32_t)nt;
    p.tile0 = (int32_t)tile0;
    const int mi = mode ? 1 : 0;
    if (!ctx->tma_smem_set[mi] || ctx->tma_smem_set_bytes[mi] < pl.smem_bytes) {
      cudaError_t e = mode == 0 ? cudaFuncSetAttribute(ua2a::ua2a_tma_kernel<0>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)ua2a::kTmaSmemMax)
                                : cudaFuncSetAttribute(ua2a::ua2a_tma_kernel<1>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)ua2a::kTmaSmemMax);
      if (e != cudaSuccess) return cuda_fail(ctx, "cudaFuncSetAttribute", e);
      ctx->tma_smem_set[mi] = true;
      ctx->tma_smem_set_bytes[mi] = ua2a::kTmaSmemMax;
    }
    for (int l = 0; l < launches; ++l) {
      p.b0 = chunked ? l : 0;
      cudaError_t le = launch_tma(mode, grid, pl.block, (size_t)pl.smem_bytes, st, p);
      if (le != cudaSuccess) return cuda_fail(ctx, "TMA kernel launch", le);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return cuda_fail(ctx, "TMA kernel launch", e);
      ctx->launches++;
    }
    return ULYSSES_A2A_OK;
  }
  VecParams p{};
  const int nin = mode == 0 ? w : w * ntensors;
  const int nout = mode == 0 ? w * ntensors : w;
  for (int k = 0; k < nin; ++k) p.in[k] = static_cast<const char*>(in[k]);
  for (int k = 0; k < nout; ++k) p.out[k] = static_cast<char*>(out[k]);
  p.S_local = S;
  p.nv = pl.row_bytes / pl.vec_bytes;
  p.srow = pl.row_pitch * ctx->elem_bytes / pl.vec_bytes;
  p.w = w;
  p.rows_per_tile = (int32_t)pl.rows_per_tile;
  p.units = (uint32_t)units;
  p.order = pl.order;
  p.tile0 = (uint32_t)tile0;
  p.r0 = (only_out >= 0 && mode == 0) ? (uint32_t)only_out : 0u;
  p.j0 = (only_out >= 0 && mode == 1) ? (uint32_t)only_out : 0u;
  p.div_T = ua2a::FastDiv((uint32_t)nt);
  p.div_nr = ua2a::FastDiv((uint32_t)nr);
  p.div_nj = ua2a::FastDiv((uint32_t)nj);
  p.div_nb = ua2a::FastDiv((uint32_t)nb);
  p.div_nv = ua2a::FastDiv((uint32_t)p.nv);
  for (int l = 0; l < launches; ++l) {
    p.b0 = chunked ? l : 0;
    cudaError_t e = launch_vec(p, pl.vec_bytes, mode, grid, pl.block, st);
    if (e != cudaSuccess) return cuda_fail(ctx, "VEC kernel launch", e);
    ctx->launches++;
  }
  return ULYSSES_A2A_OK;
}

int plan_for(ulysses_a2a_ctx* ctx, const void* const* in, void* const* out, int64_t B, int64_t S,
             int64_t H, int64_t D, int w, int mode, int chunked, ulysses_a2a_plan_t* pl,
             int64_t row_pitch = 0, int ntensors = 1) {
  std::string err;
  int rc = ua2a::make_plan(in, out, B, S, H, D, w, mode, chunked, ctx->elem_bytes, ctx->forced_path,
                           ctx->tuning, ctx->num_sms, pl, &err, row_pitch, -1, ntensors);
  if (rc) return fail(ctx, rc, err);
  return ULYSSES_A2A_OK;
}

// Test-only configuration read when a context is created; set_path and
// set_tuning override it afterwards. ULYSSES_A2A_FORCE_PATH = auto | tma | vec
// forces a copy path, ULYSSES_A2A_CTAS_PER_SM = 1..32 sets the ctas_per_sm
// knob. Returns false on a malformed value (creation then fails).
bool env_config(int* path, int* ctas) {
  if (const char* v = std::getenv("ULYSSES_A2A_FORCE_PATH")) {
    const std::string s(v);
    if (s == "auto" || s.empty()) *path = ULYSSES_A2A_PATH_AUTO;
    else if (s == "tma") *path = ULYSSES_A2A_PATH_TMA;
    else if (s == "vec") *path = ULYSSES_A2A_PATH_VEC;
    else return false;
  }
  if (const char* v = std::getenv("ULYSSES_A2A_CTAS_PER_SM")) {
    char* end = nullptr;
    const long n = std::strtol(v, &end, 10);
    if (end == v || *end != '\0' || n < 1 || n > 32) return false;
    *ctas = (int)n;
  }
  return true;
}

}  // namespace

extern "C" {

static int ua2a_impl_create(ulysses_a2a_ctx** out, int device, int elem_bytes) {
  if (out == nullptr) return ULYSSES_A2A_ERR_INVALID;
  *out = nullptr;
  if (!(elem_bytes == 1 || elem_bytes == 2 || elem_bytes == 4 || elem_bytes == 8))
    return ULYSSES_A2A_ERR_INVALID;
  int env_path = ULYSSES_A2A_PATH_AUTO, env_ctas = 0;
  if (!env_config(&env_path, &env_ctas)) return ULYSSES_A2A_ERR_INVALID;
  int count = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess || device < 0 || device >= count) {
    cudaGetLastError();
    return ULYSSES_A2A_ERR_DEVICE;
  }
  ulysses_a2a_ctx* ctx = new (std::nothrow) ulysses_a2a_ctx();
  if (!ctx) return ULYSSES_A2A_ERR_NOMEM;
  ctx->device = device;
  ctx->elem_bytes = elem_bytes;
  ctx->forced_path = env_path;
  ctx->tuning.ctas_per_sm = env_ctas;
  DeviceGuard g(device);
  if (!g.ok) {
    delete ctx;
    return ULYSSES_A2A_ERR_DEVICE;
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess || prop.major < 10) {
    delete ctx;
    return ULYSSES_A2A_ERR_DEVICE;  // built for sm_100a only
  }
  ctx->num_sms = prop.multiProcessorCount;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr) {
    delete ctx;
    return ULYSSES_A2A_ERR_CUDA;
  }
  ctx->encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  fn = nullptr;
  if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &fn, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    ctx->get_range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
  if (cudaMalloc(&ctx->d_status, 4 * sizeof(unsigned int)) != cudaSuccess) {
    cudaGetLastError();
    delete ctx;
    return ULYSSES_A2A_ERR_NOMEM;
  }
  if (cudaMemset(ctx->d_status, 0, 4 * sizeof(unsigned int)) != cudaSuccess) {
    cudaFree(ctx->d_status);
    delete ctx;
    return ULYSSES_A2A_ERR_CUDA;
  }
  *out = ctx;
  return ULYSSES_A2A_OK;
}

static int ua2a_impl_destroy(ulysses_a2a_ctx* ctx) {
  if (ctx == nullptr) return ULYSSES_A2A_OK;
  int rc = ULYSSES_A2A_OK;
  {
    DeviceGuard g(ctx->device);
    if (cudaDeviceSynchronize() != cudaSuccess) rc = ULYSSES_A2A_ERR_CUDA;
    if (ctx->d_status && cudaFree(ctx->d_status) != cudaSuccess) rc = ULYSSES_A2A_ERR_CUDA;
    if (ctx->d_stage && cudaFree(ctx->d_stage) != cudaSuccess) rc = ULYSSES_A2A_ERR_CUDA;
    if (ctx->d_window && cudaFree(ctx->d_window) != cudaSuccess) rc = ULYSSES_A2A_ERR_CUDA;
    for (auto& cs : ctx->copy_stream)
      if (cs && cudaStreamDestroy(cs) != cudaSuccess) rc = ULYSSES_A2A_ERR_CUDA;
    for (auto& ev : ctx->copy_events)
      if (ev && cudaEventDestroy(ev) != cudaSuccess) rc = ULYSSES_A2A_ERR_CUDA;
    cudaGetLastError();
  }
  delete ctx;  // the handle is consumed whatever the cleanup calls reported
  return rc;
}

namespace {

// chunked = 2: per plane, publish every rank's input plane into the window
// (the page's registered window, reused plane after plane: each copy finishes
// in stream order before the next plane overwrites it), then re-lay it out
// from the window into that plane of the outputs.
int run_windowed(ulysses_a2a_ctx* ctx, const ulysses_a2a_desc_t* d, const ulysses_a2a_plan_t& pl,
                 cudaStream_t st) {
  const int w = d->w;
  const int64_t E = ctx->elem_bytes;
  const int64_t HD = d->H * d->D;
  const size_t plane = (size_t)(d->S_local * HD * E);        // one dense plane of one slab
  const size_t slot = (plane + 255) / 256 * 256;
  const size_t need = slot * (size_t)w;
  if (ctx->window_bytes < need) {                              // grow on demand
    cudaError_t e;
    if (ctx->d_window) {
      e = cudaStreamSynchronize(st);
      if (e != cudaSuccess) return cuda_fail(ctx, "cudaStreamSynchronize (window grow)", e);
      cudaFree(ctx->d_window);
      ctx->d_window = nullptr;
      ctx->window_bytes = 0;
      for (auto& c : ctx->tma_cache) c.valid = false;       // maps may point into it
    }
    e = cudaMalloc(&ctx->d_window, need);
    if (e != cudaSuccess) {
      ctx->d_window = nullptr;
      return cuda_fail(ctx, "cudaMalloc (staging window)", e);
    }
    ctx->window_bytes = need;
  }
  std::vector<const void*> win(w);
  std::vector<void*> outb(w);
  char* wbase = static_cast<char*>(ctx->d_window);
  for (int k = 0; k < w; ++k) win[k] = wbase + slot * k;
  const int64_t pitch = pl.row_pitch;
  for (int64_t b = 0; b < d->B; ++b) {
    for (int k = 0; k < w; ++k) {
      cudaError_t e;
      if (d->mode == 0) {   // pitched [B, S, H, D] input plane -> dense window slot
        const char* src = static_cast<const char*>(d->in_slabs[k]) + (size_t)(b * d->S_local * pitch * E);
        if (pitch == HD)
          e = cudaMemcpyAsync(const_cast<void*>(win[k]), src, plane, cudaMemcpyDeviceToDevice, st);
        else
          e = cudaMemcpy2DAsync(const_cast<void*>(win[k]), (size_t)(HD * E), src, (size_t)(pitch * E),
                                (size_t)(HD * E), (size_t)d->S_local, cudaMemcpyDeviceToDevice, st);
        outb[k] = static_cast<char*>(d->out_slabs[k]) + plane * b;
      } else {              // dense [B, S*w, H/w, D] input plane -> window slot
        const char* src = static_cast<const char*>(d->in_slabs[k]) + plane * b;
        e = cudaMemcpyAsync(const_cast<void*>(win[k]), src, plane, cudaMemcpyDeviceToDevice, st);
        outb[k] = static_cast<char*>(d->out_slabs[k]) + (size_t)(b * d->S_local * pitch * E);
      }
      if (e != cudaSuccess) return cuda_fail(ctx, "cudaMemcpyAsync (publish into the window)", e);
    }
    ulysses_a2a_plan_t pb;
    int rc = plan_for(ctx, win.data(), outb.data(), 1, d->S_local, d->H, d->D, w, d->mode, 0, &pb,
                      d->mode == 1 ? pitch : 0);
    if (rc) return rc;
    rc = run_device(ctx, win.data(), outb.data(), 1, d->S_local, d->H, d->D, w, d->mode, 0, st, pb);
    if (rc) return rc;
  }
  return ULYSSES_A2A_OK;
}

}  // namespace

static int ua2a_impl_run_ex(ulysses_a2a_ctx* ctx, const ulysses_a2a_desc_t* d, void* stream) {
  if (ctx == nullptr) return ULYSSES_A2A_ERR_INVALID;
  ctx->last_error.clear();
  if (d == nullptr) return fail(ctx, ULYSSES_A2A_ERR_INVALID, "descriptor is NULL");
  if (d->ntensors < 0 || d->row_pitch < 0)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "descriptor: ntensors and row_pitch must be >= 0");
  const int T = d->ntensors > 1 ? d->ntensors : 1;
  ulysses_a2a_plan_t pl;
  int rc = plan_for(ctx, d->in_slabs, d->out_slabs, d->B, d->S_local, d->H, d->D, d->w, d->mode,
                    d->chunked, &pl, d->row_pitch, T);
  if (rc) return rc;
  if (pl.units == 0) return ULYSSES_A2A_OK;  // empty: nothing to do
  DeviceGuard g(ctx->device);
  if (!g.ok) return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "cannot select the context's device");
  // one [B, S*w, H/w, D] slab, and one (pitched, T-packed) [B, S, (T,) H, D] slab
  const int64_t dense_bytes = pl.payload_bytes / ((int64_t)d->w * T);
  const int64_t strided_bytes = ((d->B * d->S_local - 1) * pl.row_pitch + (int64_t)T * d->H * d->D) *
                                (int64_t)ctx->elem_bytes;
  const int nin = d->mode == 0 ? d->w : d->w * T;
  const int nout = d->mode == 0 ? d->w * T : d->w;
  rc = check_residency(ctx, d->in_slabs, nin, d->mode == 0 ? strided_bytes : dense_bytes, "input");
  if (rc) return rc;
  rc = check_residency(ctx, reinterpret_cast<const void* const*>(d->out_slabs), nout,
                       d->mode == 0 ? dense_bytes : strided_bytes, "output");
  if (rc) return rc;
  if (d->chunked == ULYSSES_A2A_CHUNKED_WINDOW)
    return run_windowed(ctx, d, pl, static_cast<cudaStream_t>(stream));
  return run_device(ctx, d->in_slabs, d->out_slabs, d->B, d->S_local, d->H, d->D, d->w, d->mode,
                    d->chunked, static_cast<cudaStream_t>(stream), pl, 0, -1, -1, T);
}

static int ua2a_impl_run(ulysses_a2a_ctx* ctx, const void* const* in_slabs, void* const* out_slabs,
                    int64_t B, int64_t S_local, int64_t H, int64_t D, int w, int mode, int chunked,
                    void* stream) {
  ulysses_a2a_desc_t d{};
  d.in_slabs = in_slabs;
  d.out_slabs = out_slabs;
  d.B = B;
  d.S_local = S_local;
  d.H = H;
  d.D = D;
  d.w = w;
  d.mode = mode;
  d.chunked = chunked;
  d.row_pitch = 0;
  return ulysses_a2a_run_ex(ctx, &d, stream);
}

static int ua2a_impl_run_host(ulysses_a2a_ctx* ctx, const void* const* in_slabs, void* const* out_slabs,
                         int64_t B, int64_t S_local, int64_t H, int64_t D, int w, int mode,
                         int chunked, void* stream) {
  if (ctx == nullptr) return ULYSSES_A2A_ERR_INVALID;
  ctx->last_error.clear();
  // validate the host pointers (overlap, sizes) before touching the device
  if (chunked == ULYSSES_A2A_CHUNKED_WINDOW)
    return fail(ctx, ULYSSES_A2A_ERR_UNSUPPORTED,
                "the host-buffer path stages through its own buffers: chunked must be 0 or 1");
  ulysses_a2a_plan_t host_pl;
  int rc = plan_for(ctx, in_slabs, out_slabs, B, S_local, H, D, w, mode, chunked, &host_pl);
  if (rc) return rc;
  if (host_pl.units == 0) return ULYSSES_A2A_OK;  // empty: nothing to do
  DeviceGuard g(ctx->device);
  if (!g.ok) return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "cannot select the context's device");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t slab_bytes = host_pl.payload_bytes / w;
  const size_t slot = ((size_t)slab_bytes + 255) / 256 * 256;
  const size_t need = slot * 2 * (size_t)w;
  if (ctx->stage_bytes < need) {
    if (ctx->d_stage) {
      cudaError_t e = cudaDeviceSynchronize();
      if (e != cudaSuccess) return cuda_fail(ctx, "cudaDeviceSynchronize", e);
      cudaFree(ctx->d_stage);
      ctx->d_stage = nullptr;
      ctx->stage_bytes = 0;
      for (auto& c : ctx->tma_cache) c.valid = false;  // maps may point into the old buffer
    }
    cudaError_t e = cudaMalloc(&ctx->d_stage, need);
    if (e != cudaSuccess) {
      ctx->d_stage = nullptr;
      return cuda_fail(ctx, "cudaMalloc (host-path staging)", e);
    }
    ctx->stage_bytes = need;
  }
  for (int k = 0; k < 2; ++k) {
    if (ctx->copy_stream[k] == nullptr) {
      cudaError_t e = cudaStreamCreateWithFlags(&ctx->copy_stream[k], cudaStreamNonBlocking);
      if (e != cudaSuccess) {
        ctx->copy_stream[k] = nullptr;
        return cuda_fail(ctx, "cudaStreamCreate (host-path copies)", e);
      }
    }
  }
  while (ctx->copy_events.size() < (size_t)(1 + 2 * ua2a::kHostMaxChunks)) {
    cudaEvent_t ev = nullptr;
    cudaError_t e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(ctx, "cudaEventCreate (host-path copies)", e);
    ctx->copy_events.push_back(ev);
  }
  std::vector<const void*> din(w);
  std::vector<void*> dout(w);
  char* base = static_cast<char*>(ctx->d_stage);
  for (int k = 0; k < w; ++k) {
    din[k] = base + slot * k;
    dout[k] = base + slot * (w + k);
  }
  ulysses_a2a_plan_t pl;
  rc = plan_for(ctx, din.data(), dout.data(), B, S_local, H, D, w, mode, chunked, &pl);
  if (rc) return rc;

  // Pipeline over sequence chunks: the H2D copies of chunk c+1 (copy stream 0),
  // the kernel of chunk c (the caller's stream) and the D2H copies of chunk
  // c-1 (copy stream 1) run at once, so PCIe carries both directions together.
  // A chunk is a tile-aligned row range [s0, s1) of every (b, j) block; its
  // bytes on each side are strided blocks moved by one 2-D copy per slab/plane.
  const int64_t T = pl.tiles_per_block, rows = pl.rows_per_tile, E = ctx->elem_bytes;
  const int64_t L = (H / w) * D;             // elements per run
  // Chunk boundaries (in tiles): equal chunks. (Shorter first and last chunks,
  // to shrink the pipeline's fill and drain, measured no better.)
  int64_t nchunks = ctx->tuning.host_chunks > 0 ? ctx->tuning.host_chunks : ua2a::kHostDefaultChunks;
  if (pl.payload_bytes < ua2a::kHostChunkMinBytes) nchunks = 1;
  if (nchunks > T) nchunks = T;
  std::vector<int64_t> bounds;  // chunk c covers tiles [bounds[c], bounds[c+1])
  for (int64_t c = 0; c <= nchunks; ++c) bounds.push_back(T * c / nchunks);
  cudaStream_t sh = ctx->copy_stream[0], sd = ctx->copy_stream[1];
  cudaEvent_t* ev = ctx->copy_events.data();  // [0]: start; [1 + 2c]: H2D; [2 + 2c]: kernel
  cudaError_t e = cudaEventRecord(ev[0], st);  // copies start after earlier work on `stream`
  if (e == cudaSuccess) e = cudaStreamWaitEvent(sh, ev[0], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(sd, ev[0], 0);
  if (e != cudaSuccess) return cuda_fail(ctx, "stream ordering", e);
  const size_t plane_s = (size_t)(S_local * H * D * E);   // [B, S, H, D] plane
  const size_t row_s = (size_t)(H * D * E);
  const size_t plane_g = (size_t)(w * S_local * L * E);   // [B, S*w, H/w, D] plane
  const size_t block_g = (size_t)(S_local * L * E);       // one j block of it
  const size_t row_g = (size_t)(L * E);
  auto copy_rows = [&](bool h2d, int64_t s0, int64_t n, cudaStream_t cs) -> cudaError_t {
    // mode 0 reads the [B,S,H,D] side and writes the [B,S*w,H/w,D] side;
    // mode 1 the reverse
    const bool strided_side = (mode == 0) == h2d;
    for (int k = 0; k < w; ++k) {
      const char* src_base = static_cast<const char*>(h2d ? in_slabs[k] : dout[k]);
      char* dst_base = static_cast<char*>(h2d ? const_cast<void*>(din[k]) : out_slabs[k]);
      cudaMemcpyKind kind = h2d ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost;
      cudaError_t r;
      if (strided_side) {
        // rows [s0, s0+n) of every plane: B blocks of n*H*D*E bytes, plane apart
        const size_t off = (size_t)s0 * row_s;
        r = cudaMemcpy2DAsync(dst_base + off, plane_s, src_base + off, plane_s, (size_t)n * row_s,
                              (size_t)B, kind, cs);
      } else {
        // rows [s0, s0+n) of every (b, j) block: per plane, w blocks S*L*E apart
        r = cudaSuccess;
        for (int64_t b = 0; b < B && r == cudaSuccess; ++b) {
          const size_t off = b * plane_g + (size_t)s0 * row_g;
          r = cudaMemcpy2DAsync(dst_base + off, block_g, src_base + off, block_g, (size_t)n * row_g,
                                (size_t)w, kind, cs);
        }
      }
      if (r != cudaSuccess) return r;
    }
    return cudaSuccess;
  };
  for (int64_t c = 0; c < nchunks; ++c) {
    const int64_t t0 = bounds[c];
    const int64_t nt = bounds[c + 1] - t0;
    if (nt <= 0) continue;
    const int64_t s0 = t0 * rows;
    const int64_t s1 = (t0 + nt) * rows < S_local ? (t0 + nt) * rows : S_local;
    e = copy_rows(true, s0, s1 - s0, sh);
    if (e == cudaSuccess) e = cudaEventRecord(ev[1 + 2 * c], sh);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev[1 + 2 * c], 0);
    if (e != cudaSuccess) return cuda_fail(ctx, "host-path H2D copy", e);
    rc = run_device(ctx, din.data(), dout.data(), B, S_local, H, D, w, mode, chunked, st, pl, t0, nt);
    if (rc) return rc;
    e = cudaEventRecord(ev[2 + 2 * c], st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sd, ev[2 + 2 * c], 0);
    if (e == cudaSuccess) e = copy_rows(false, s0, s1 - s0, sd);
    if (e != cudaSuccess) return cuda_fail(ctx, "host-path D2H copy", e);
  }
  e = cudaStreamSynchronize(sd);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(ctx, "cudaStreamSynchronize", e);
  return ULYSSES_A2A_OK;
}

const char* ulysses_a2a_last_error(const ulysses_a2a_ctx* ctx) {
  if (ctx == nullptr) return "NULL context";
  return ctx->last_error.c_str();
}

static int ua2a_impl_status(ulysses_a2a_ctx* ctx, void* stream) {
  if (ctx == nullptr) return ULYSSES_A2A_ERR_INVALID;
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(ctx, "cudaStreamSynchronize", e);
  unsigned int h[4] = {0, 0, 0, 0};
  e = cudaMemcpy(h, ctx->d_status, sizeof(h), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(ctx, "cudaMemcpy (status word)", e);
  if (h[0] == 0) return ULYSSES_A2A_OK;
  e = cudaMemset(ctx->d_status, 0, sizeof(h));
  if (e != cudaSuccess) return cuda_fail(ctx, "cudaMemset (status word)", e);
  char buf[160];
  std::snprintf(buf, sizeof(buf),
                "a TMA wait gave up (flags=0x%x, block %u, tile %u)%s", h[0],
                h[1] ? h[1] - 1 : 0u, h[2],
                (h[0] & ua2a::kStatusDrainTimeout) ? "; draining also timed out" : "");
  return fail(ctx, ULYSSES_A2A_ERR_TIMEOUT, buf);
}

static int ua2a_impl_selftest_wait_timeout(ulysses_a2a_ctx* ctx, uint32_t limit_us, void* stream) {
  if (ctx == nullptr) return ULYSSES_A2A_ERR_INVALID;
  if (limit_us < 1 || limit_us > 2000000)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "limit_us must be in [1, 2000000]");
  DeviceGuard g(ctx->device);
  if (!g.ok) return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "cannot select the context's device");
  ua2a::ua2a_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      ctx->d_status, (uint64_t)limit_us * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(ctx, "self-test kernel launch", e);
  ctx->launches++;
  return ULYSSES_A2A_OK;
}

static int ua2a_impl_set_path(ulysses_a2a_ctx* ctx, int path) {
  if (ctx == nullptr) return ULYSSES_A2A_ERR_INVALID;
  if (path < ULYSSES_A2A_PATH_AUTO || path > ULYSSES_A2A_PATH_VEC)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "unknown path");
  ctx->forced_path = path;
  return ULYSSES_A2A_OK;
}

static int ua2a_impl_set_tuning(ulysses_a2a_ctx* ctx, const ulysses_a2a_tuning_t* t) {
  if (ctx == nullptr) return ULYSSES_A2A_ERR_INVALID;
  ua2a::Tuning tu;
  std::string err;
  if (!ua2a::tuning_from(t, &tu, &err)) return fail(ctx, ULYSSES_A2A_ERR_INVALID, err);
  ctx->tuning = tu;
  return ULYSSES_A2A_OK;
}

static int ua2a_impl_get_settings(const ulysses_a2a_ctx* ctx, int32_t* path,
                                  ulysses_a2a_tuning_t* t) {
  if (ctx == nullptr) return ULYSSES_A2A_ERR_INVALID;
  if (path) *path = ctx->forced_path;
  if (t) {
    const ua2a::Tuning& u = ctx->tuning;
    t->rows_per_tile = u.rows_per_tile;
    t->ctas_per_sm = u.ctas_per_sm;
    t->stages = u.stages;
    t->lookahead = u.lookahead;
    t->producers = u.producers;
    t->order = u.order;
    t->chunk_units = u.chunk_units;
    t->host_chunks = u.host_chunks;
  }
  return ULYSSES_A2A_OK;
}

uint64_t ulysses_a2a_launch_count(const ulysses_a2a_ctx* ctx) {
  return ctx ? ctx->launches : 0;
}

static int ua2a_impl_plan_ex(const ulysses_a2a_desc_t* d, int elem_bytes, int forced_path,
                        const ulysses_a2a_tuning_t* tuning, int num_sms, ulysses_a2a_plan_t* out,
                        char* err, size_t errlen) {
  ua2a::Tuning t;
  std::string msg;
  int rc = ULYSSES_A2A_OK;
  if (d == nullptr) {
    msg = "descriptor is NULL";
    rc = ULYSSES_A2A_ERR_INVALID;
  } else if (d->ntensors < 0 || d->row_pitch < 0) {
    msg = "descriptor: ntensors and row_pitch must be >= 0";
    rc = ULYSSES_A2A_ERR_INVALID;
  } else if (!ua2a::tuning_from(tuning, &t, &msg)) {
    rc = ULYSSES_A2A_ERR_INVALID;
  } else {
    rc = ua2a::make_plan(d->in_slabs, d->out_slabs, d->B, d->S_local, d->H, d->D, d->w, d->mode,
                         d->chunked, elem_bytes, forced_path, t, num_sms, out, &msg, d->row_pitch,
                         -1, d->ntensors > 1 ? d->ntensors : 1);
  }
  if (err && errlen) std::snprintf(err, errlen, "%s", rc ? msg.c_str() : "");
  return rc;
}

static int ua2a_impl_plan(const void* const* in_slabs, void* const* out_slabs, int64_t B,
                     int64_t S_local, int64_t H, int64_t D, int w, int mode, int chunked,
                     int elem_bytes, int forced_path, const ulysses_a2a_tuning_t* tuning,
                     int num_sms, ulysses_a2a_plan_t* out, char* err, size_t errlen) {
  ua2a::Tuning t;
  std::string msg;
  int rc = ULYSSES_A2A_OK;
  if (!ua2a::tuning_from(tuning, &t, &msg))
    rc = ULYSSES_A2A_ERR_INVALID;
  else
    rc = ua2a::make_plan(in_slabs, out_slabs, B, S_local, H, D, w, mode, chunked, elem_bytes,
                         forced_path, t, num_sms, out, &msg);
  if (err && errlen) {
    std::snprintf(err, errlen, "%s", rc ? msg.c_str() : "");
  }
  return rc;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Multi-GPU exchange through published windows (ulysses_a2a_peer_*).
//
// Each rank owns one device window that the other ranks map: CUDA IPC between
// processes, the plain address inside one process. A call publishes the local
// input slab into the own window (a w = 1 re-layout, i.e. a copy that drops any
// row pitch), and after the caller's barrier pulls this rank's output slab out
// of all w windows with the VEC kernel restricted to that one output slab, so
// the bytes crossing NVLink are read by the GPU that needs them and written to
// its own memory. The barriers are left to the caller: no kernel here waits on
// another GPU.
// ---------------------------------------------------------------------------

namespace {

constexpr uint32_t kPeerMagic = 0x50324155u;  // "UA2P"
constexpr uint32_t kPeerVersion = 1;

// The record one rank hands to the others (ULYSSES_A2A_PEER_HANDLE_BYTES).
struct PeerRecord {
  uint32_t magic;
  uint32_t version;
  uint64_t process_nonce;  // random per process: with pid, tells "same process"
  int32_t rank;
  int32_t world;
  int32_t device;          // owner's device ordinal (meaningful in its process)
  int32_t elem_bytes;
  uint64_t window_bytes;
  uint64_t base;           // owner's window address (used in the same process)
  uint64_t pid;
  cudaIpcMemHandle_t ipc;  // 64 bytes; valid if ipc_ok
  int32_t ipc_ok;
  int32_t pad;
};
static_assert(sizeof(PeerRecord) == ULYSSES_A2A_PEER_HANDLE_BYTES, "peer record size");

uint64_t process_nonce() {
  static std::once_flag once;
  static uint64_t nonce = 0;
  std::call_once(once, [] {
    uint64_t v = (uint64_t)std::chrono::steady_clock::now().time_since_epoch().count();
    v ^= (uint64_t)getpid() << 17;
    v ^= (uint64_t)(uintptr_t)&nonce;
    try {  // no exception may leave the C ABI
      std::random_device rd;
      v ^= ((uint64_t)rd() << 32) ^ (uint64_t)rd();
    } catch (...) {
    }
    nonce = v ? v : 1;
  });
  return nonce;
}

}  // namespace

struct ulysses_a2a_peer {
  ulysses_a2a_ctx* ctx = nullptr;
  int rank = 0, world = 1;
  size_t window_bytes = 0;
  void* own = nullptr;
  std::vector<void*> bases;        // window of rank k as mapped here
  std::vector<char> ipc_opened;    // 1 where cudaIpcOpenMemHandle made the mapping
  bool open = false;
};

namespace {

void peer_unmap(ulysses_a2a_peer* p, int* rc) {
  for (int k = 0; k < p->world; ++k) {
    if (k == p->rank) continue;
    if (p->ipc_opened[k] && p->bases[k] && cudaIpcCloseMemHandle(p->bases[k]) != cudaSuccess) {
      cudaGetLastError();
      if (rc) *rc = ULYSSES_A2A_ERR_CUDA;
    }
    p->ipc_opened[k] = 0;
    p->bases[k] = nullptr;
  }
  p->open = false;
}

}  // namespace

extern "C" {

static int ua2a_impl_peer_create(ulysses_a2a_ctx* ctx, int rank, int world, size_t window_bytes,
                            ulysses_a2a_peer** out, void* handle_out) {
  if (out) *out = nullptr;
  if (ctx == nullptr) return ULYSSES_A2A_ERR_INVALID;
  ctx->last_error.clear();
  if (out == nullptr || handle_out == nullptr)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_create: out or handle_out is NULL");
  if (world < 1 || world > ULYSSES_A2A_MAX_W || rank < 0 || rank >= world)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_create: need 1 <= world <= 64, 0 <= rank < world");
  if (window_bytes < 1) return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_create: window_bytes must be >= 1");
  DeviceGuard g(ctx->device);
  if (!g.ok) return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "cannot select the context's device");
  ulysses_a2a_peer* p = new (std::nothrow) ulysses_a2a_peer();
  if (!p) return fail(ctx, ULYSSES_A2A_ERR_NOMEM, "peer_create: host allocation failed");
  p->ctx = ctx;
  p->rank = rank;
  p->world = world;
  p->window_bytes = window_bytes;
  p->bases.assign(world, nullptr);
  p->ipc_opened.assign(world, 0);
  cudaError_t e = cudaMalloc(&p->own, window_bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    delete p;
    return fail(ctx, ULYSSES_A2A_ERR_NOMEM, "peer_create: cudaMalloc of the window failed");
  }
  p->bases[rank] = p->own;
  PeerRecord r;
  std::memset(&r, 0, sizeof(r));
  r.magic = kPeerMagic;
  r.version = kPeerVersion;
  r.process_nonce = process_nonce();
  r.rank = rank;
  r.world = world;
  r.device = ctx->device;
  r.elem_bytes = ctx->elem_bytes;
  r.window_bytes = window_bytes;
  r.base = (uint64_t)(uintptr_t)p->own;
  r.pid = (uint64_t)getpid();
  // a window that cannot be exported still serves ranks in this process
  r.ipc_ok = cudaIpcGetMemHandle(&r.ipc, p->own) == cudaSuccess ? 1 : 0;
  if (!r.ipc_ok) cudaGetLastError();
  std::memcpy(handle_out, &r, sizeof(r));
  *out = p;
  return ULYSSES_A2A_OK;
}

static int ua2a_impl_peer_open(ulysses_a2a_peer* p, const void* handles) {
  if (p == nullptr) return ULYSSES_A2A_ERR_INVALID;
  ulysses_a2a_ctx* ctx = p->ctx;
  ctx->last_error.clear();
  if (handles == nullptr) return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_open: handles is NULL");
  if (p->open) return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_open: already open");
  std::vector<PeerRecord> recs(p->world);
  std::memcpy(recs.data(), handles, sizeof(PeerRecord) * (size_t)p->world);
  const uint64_t nonce = process_nonce();
  const uint64_t pid = (uint64_t)getpid();
  // check every record before mapping anything
  for (int k = 0; k < p->world; ++k) {
    const PeerRecord& r = recs[k];
    const std::string who = "peer_open: record " + std::to_string(k);
    if (r.magic != kPeerMagic || r.version != kPeerVersion)
      return fail(ctx, ULYSSES_A2A_ERR_INVALID, who + " is not a peer record of this library version");
    if (r.rank != k || r.world != p->world)
      return fail(ctx, ULYSSES_A2A_ERR_INVALID, who + " carries rank " + std::to_string(r.rank) +
                                                    " of world " + std::to_string(r.world));
    if (r.elem_bytes != ctx->elem_bytes || r.window_bytes != (uint64_t)p->window_bytes)
      return fail(ctx, ULYSSES_A2A_ERR_INVALID, who + ": element size or window size differs");
    const bool local = r.process_nonce == nonce && r.pid == pid;
    if (k == p->rank && !(local && r.base == (uint64_t)(uintptr_t)p->own))
      return fail(ctx, ULYSSES_A2A_ERR_INVALID, who + " is not this peer's own record");
    if (k != p->rank && !local && !r.ipc_ok)
      return fail(ctx, ULYSSES_A2A_ERR_DEVICE, who + ": its window could not be exported (CUDA IPC)");
  }
  DeviceGuard g(ctx->device);
  if (!g.ok) return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "cannot select the context's device");
  for (int k = 0; k < p->world; ++k) {
    if (k == p->rank) continue;
    const PeerRecord& r = recs[k];
    const bool local = r.process_nonce == nonce && r.pid == pid;
    cudaError_t e = cudaSuccess;
    if (local) {
      if (r.device != ctx->device) {
        int can = 0;
        e = cudaDeviceCanAccessPeer(&can, ctx->device, r.device);
        if (e == cudaSuccess && !can) {
          peer_unmap(p, nullptr);
          return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "peer_open: device " + std::to_string(ctx->device) +
                                                       " cannot access device " + std::to_string(r.device));
        }
        if (e == cudaSuccess) {
          e = cudaDeviceEnablePeerAccess(r.device, 0);
          if (e == cudaErrorPeerAccessAlreadyEnabled) {
            cudaGetLastError();
            e = cudaSuccess;
          }
        }
      }
      if (e == cudaSuccess) p->bases[k] = reinterpret_cast<void*>((uintptr_t)r.base);
    } else {
      void* ptr = nullptr;
      e = cudaIpcOpenMemHandle(&ptr, r.ipc, cudaIpcMemLazyEnablePeerAccess);
      if (e == cudaSuccess) {
        p->bases[k] = ptr;
        p->ipc_opened[k] = 1;
      }
    }
    if (e != cudaSuccess) {
      cudaGetLastError();
      peer_unmap(p, nullptr);
      return cuda_fail(ctx, ("peer_open: mapping the window of rank " + std::to_string(k)).c_str(), e);
    }
  }
  p->open = true;
  return ULYSSES_A2A_OK;
}

static int ua2a_impl_peer_publish(ulysses_a2a_peer* p, const void* in_local, int64_t B, int64_t S_local,
                             int64_t H, int64_t D, int mode, int64_t row_pitch, void* stream) {
  if (p == nullptr) return ULYSSES_A2A_ERR_INVALID;
  ulysses_a2a_ctx* ctx = p->ctx;
  ctx->last_error.clear();
  const int w = p->world;
  if (mode != 0 && mode != 1) return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_publish: mode must be 0 or 1");
  if (B < 0 || S_local < 0 || H < 0 || D < 0 || row_pitch < 0)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_publish: sizes and row_pitch must be >= 0");
  if (H % w != 0) return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_publish: H not divisible by the world size");
  if (mode == 1 && row_pitch != 0)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_publish: a mode-1 input is dense (row_pitch 0)");
  // the copy, as a one-rank re-layout: mode 0 keeps [B, S, H, D] (dropping the
  // pitch); mode 1 copies [B, S*w, H/w, D]
  const int64_t S1 = mode == 0 ? S_local : S_local * w;
  const int64_t H1 = mode == 0 ? H : H / w;
  if (in_local == p->own && (row_pitch == 0 || row_pitch == H1 * D)) {
    // the slab was written into the window in place: nothing to copy
    int64_t bytes = 0;
    if (ua2a::mul_overflows(B, S1, &bytes) || ua2a::mul_overflows(bytes, H1, &bytes) ||
        ua2a::mul_overflows(bytes, D, &bytes) ||
        ua2a::mul_overflows(bytes, (int64_t)ctx->elem_bytes, &bytes) ||
        (uint64_t)bytes > (uint64_t)p->window_bytes)
      return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_publish: the slab exceeds the window");
    return ULYSSES_A2A_OK;
  }
  const void* in[1] = {in_local};
  void* out[1] = {p->own};
  ulysses_a2a_plan_t pl;
  int rc = plan_for(ctx, in, out, B, S1, H1, D, 1, 0, 0, &pl, row_pitch);
  if (rc) return rc;
  if (pl.units == 0) return ULYSSES_A2A_OK;
  if ((uint64_t)pl.payload_bytes > (uint64_t)p->window_bytes)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_publish: the slab (" + std::to_string(pl.payload_bytes) +
                                                  " bytes) exceeds the window (" +
                                                  std::to_string(p->window_bytes) + " bytes)");
  DeviceGuard g(ctx->device);
  if (!g.ok) return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "cannot select the context's device");
  const int64_t in_bytes = ((B * S1 - 1) * pl.row_pitch + H1 * D) * (int64_t)ctx->elem_bytes;
  rc = check_residency(ctx, in, 1, in_bytes, "input");
  if (rc) return rc;
  return run_device(ctx, in, out, B, S1, H1, D, 1, 0, 0, static_cast<cudaStream_t>(stream), pl);
}

static int ua2a_impl_peer_pull(ulysses_a2a_peer* p, void* out_local, int64_t B, int64_t S_local, int64_t H,
                          int64_t D, int mode, int64_t row_pitch, void* stream) {
  if (p == nullptr) return ULYSSES_A2A_ERR_INVALID;
  ulysses_a2a_ctx* ctx = p->ctx;
  ctx->last_error.clear();
  if (!p->open) return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_pull: the peer windows are not open");
  const int w = p->world;
  if (mode == 0 && row_pitch != 0)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_pull: a mode-0 output is dense (row_pitch 0)");
  std::vector<void*> outs(w, nullptr);
  outs[p->rank] = out_local;
  std::string err;
  ulysses_a2a_plan_t pl;
  int rc = ua2a::make_plan(p->bases.data(), outs.data(), B, S_local, H, D, w, mode, 0, ctx->elem_bytes,
                           ULYSSES_A2A_PATH_VEC, ctx->tuning, ctx->num_sms, &pl, &err, row_pitch,
                           p->rank);
  if (rc) return fail(ctx, rc, "peer_pull: " + err);
  if (pl.units == 0) return ULYSSES_A2A_OK;
  if ((uint64_t)pl.payload_bytes > (uint64_t)p->window_bytes)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_pull: the slab (" + std::to_string(pl.payload_bytes) +
                                                  " bytes) exceeds the windows (" +
                                                  std::to_string(p->window_bytes) + " bytes)");
  DeviceGuard g(ctx->device);
  if (!g.ok) return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "cannot select the context's device");
  const int64_t out_bytes = mode == 0 ? pl.payload_bytes
                                      : ((B * S_local - 1) * pl.row_pitch + H * D) * (int64_t)ctx->elem_bytes;
  const void* o[1] = {out_local};
  rc = check_residency(ctx, o, 1, out_bytes, "output");
  if (rc) return rc;
  return run_device(ctx, p->bases.data(), outs.data(), B, S_local, H, D, w, mode, 0,
                    static_cast<cudaStream_t>(stream), pl, 0, -1, p->rank);
}

void* ulysses_a2a_peer_window(const ulysses_a2a_peer* p, int rank) {
  if (p == nullptr || rank < 0 || rank >= p->world) return nullptr;
  return p->bases[rank];
}

size_t ulysses_a2a_peer_window_bytes(const ulysses_a2a_peer* p) {
  return p ? p->window_bytes : 0;
}

static int ua2a_impl_peer_close(ulysses_a2a_peer* p) {
  if (p == nullptr) return ULYSSES_A2A_ERR_INVALID;
  if (!p->open) return ULYSSES_A2A_OK;
  int rc = ULYSSES_A2A_OK;
  DeviceGuard g(p->ctx->device);
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    rc = ULYSSES_A2A_ERR_CUDA;
  }
  peer_unmap(p, &rc);
  return rc;
}

static int ua2a_impl_peer_destroy(ulysses_a2a_peer* p) {
  if (p == nullptr) return ULYSSES_A2A_OK;
  int rc = ulysses_a2a_peer_close(p);
  {
    DeviceGuard g(p->ctx->device);
    if (p->own && cudaFree(p->own) != cudaSuccess) {
      cudaGetLastError();
      rc = ULYSSES_A2A_ERR_CUDA;
    }
  }
  delete p;  // consumed whatever the cleanup calls reported
  return rc;
}

}  // extern "C"

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
// one record per kernel launch of a call (a chunked call launches once per
// plane), held by every GPU that loads this library until the process exits.
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
  std::once_flag once;
  int rc = ULYSSES_A2A_OK;
  char why[96] = {0};
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

// Once per device, with that device current: resolve the array's device address
// (the symbol itself is only a host-side stand-in) and set the kernels' shared
// memory limit.
void noalloc_setup(NoAllocDevice& st, int dev) {
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major < 10) {
    cudaGetLastError();
    st.rc = ULYSSES_A2A_ERR_DEVICE;
    std::snprintf(st.why, sizeof(st.why), "device %d is not an sm_100 GPU", dev);
    return;
  }
  st.num_sms = prop.multiProcessorCount;
  void* addr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&addr, ua2a_noalloc_scratch);
  if (e != cudaSuccess || addr == nullptr) {
    cudaGetLastError();
    st.rc = ULYSSES_A2A_ERR_CUDA;
    std::snprintf(st.why, sizeof(st.why), "cudaGetSymbolAddress failed: %s", cudaGetErrorName(e));
    return;
  }
  st.scratch = static_cast<unsigned int*>(addr);
  if (cudaFuncSetAttribute(ua2a::ua2a_tma_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)ua2a::kTmaSmemMax) != cudaSuccess ||
      cudaFuncSetAttribute(ua2a::ua2a_tma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)ua2a::kTmaSmemMax) != cudaSuccess) {
    cudaGetLastError();
    st.rc = ULYSSES_A2A_ERR_CUDA;
    std::snprintf(st.why, sizeof(st.why), "cudaFuncSetAttribute failed");
  }
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
  std::call_once(st.once, noalloc_setup, std::ref(st), dev);
  if (st.rc != ULYSSES_A2A_OK) {
    if (err && errlen) std::snprintf(err, errlen, "%s", st.why);
    return st.rc;
  }

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
  const int slots = pl.launches;
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
  // the records of this call start at zero (the array keeps the previous call's)
  cudaError_t e = cudaMemsetAsync(st.scratch, 0, sizeof(unsigned int) * kNoAllocSlotWords * slots, st_);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA, "cudaMemsetAsync of the status records failed");
  }
  const int64_t nb = chunked ? 1 : B;
  if (pl.path == ULYSSES_A2A_PATH_TMA) {
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
  } else {
    VecParams p{};
    for (int k = 0; k < w; ++k) {
      p.in[k] = static_cast<const char*>(in_slabs[k]);
      p.out[k] = static_cast<char*>(out_slabs[k]);
    }
    p.S_local = S_local;
    p.nv = pl.row_bytes / pl.vec_bytes;
    p.srow = pl.row_pitch * elem_bytes / pl.vec_bytes;
    p.w = w;
    p.rows_per_tile = (int32_t)pl.rows_per_tile;
    p.units = (uint32_t)pl.units;
    p.order = pl.order;
    p.div_T = ua2a::FastDiv((uint32_t)pl.tiles_per_block);
    p.div_nr = ua2a::FastDiv((uint32_t)w);
    p.div_nj = ua2a::FastDiv((uint32_t)w);
    p.div_nb = ua2a::FastDiv((uint32_t)nb);
    p.div_nv = ua2a::FastDiv((uint32_t)p.nv);
    for (int l = 0; l < pl.launches; ++l) {
      p.b0 = chunked ? l : 0;
      e = launch_vec(p, pl.vec_bytes, mode, pl.grid, pl.block, st_);
      if (e != cudaSuccess)
        return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA, "VEC kernel launch failed (plane %lld)", l);
    }
  }
  if (!wait) return ULYSSES_A2A_OK;
  e = cudaStreamSynchronize(st_);
  if (e != cudaSuccess)
    return noalloc_report(err, errlen, ULYSSES_A2A_ERR_CUDA, "cudaStreamSynchronize failed");
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

// ---------------------------------------------------------------------------
// The exported entry points: no exception may cross the C ABI. A failed host
// allocation inside the library becomes ULYSSES_A2A_ERR_NOMEM, any other
// exception ULYSSES_A2A_ERR_INTERNAL.
// ---------------------------------------------------------------------------

namespace {

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

}  // namespace

extern "C" {

int ulysses_a2a_create(ulysses_a2a_ctx** out, int device, int elem_bytes) {
  return no_throw([&] { return ua2a_impl_create(out, device, elem_bytes); });
}

int ulysses_a2a_destroy(ulysses_a2a_ctx* ctx) {
  return no_throw([&] { return ua2a_impl_destroy(ctx); });
}

int ulysses_a2a_run_ex(ulysses_a2a_ctx* ctx, const ulysses_a2a_desc_t* d, void* stream) {
  return no_throw([&] { return ua2a_impl_run_ex(ctx, d, stream); });
}

int ulysses_a2a_run(ulysses_a2a_ctx* ctx, const void* const* in_slabs, void* const* out_slabs,
                    int64_t B, int64_t S_local, int64_t H, int64_t D, int w, int mode, int chunked,
                    void* stream) {
  return no_throw([&] { return ua2a_impl_run(ctx, in_slabs, out_slabs, B, S_local, H, D, w, mode,
                                             chunked, stream); });
}

int ulysses_a2a_run_host(ulysses_a2a_ctx* ctx, const void* const* in_slabs, void* const* out_slabs,
                         int64_t B, int64_t S_local, int64_t H, int64_t D, int w, int mode,
                         int chunked, void* stream) {
  return no_throw([&] { return ua2a_impl_run_host(ctx, in_slabs, out_slabs, B, S_local, H, D, w,
                                                  mode, chunked, stream); });
}

int ulysses_a2a_status(ulysses_a2a_ctx* ctx, void* stream) {
  return no_throw([&] { return ua2a_impl_status(ctx, stream); });
}

int ulysses_a2a_selftest_wait_timeout(ulysses_a2a_ctx* ctx, uint32_t limit_us, void* stream) {
  return no_throw([&] { return ua2a_impl_selftest_wait_timeout(ctx, limit_us, stream); });
}

int ulysses_a2a_set_path(ulysses_a2a_ctx* ctx, int path) {
  return no_throw([&] { return ua2a_impl_set_path(ctx, path); });
}

int ulysses_a2a_set_tuning(ulysses_a2a_ctx* ctx, const ulysses_a2a_tuning_t* t) {
  return no_throw([&] { return ua2a_impl_set_tuning(ctx, t); });
}

int ulysses_a2a_plan_ex(const ulysses_a2a_desc_t* d, int elem_bytes, int forced_path,
                        const ulysses_a2a_tuning_t* tuning, int num_sms, ulysses_a2a_plan_t* out,
                        char* err, size_t errlen) {
  return no_throw([&] { return ua2a_impl_plan_ex(d, elem_bytes, forced_path, tuning, num_sms, out,
                                                 err, errlen); });
}

int ulysses_a2a_plan(const void* const* in_slabs, void* const* out_slabs, int64_t B,
                     int64_t S_local, int64_t H, int64_t D, int w, int mode, int chunked,
                     int elem_bytes, int forced_path, const ulysses_a2a_tuning_t* tuning,
                     int num_sms, ulysses_a2a_plan_t* out, char* err, size_t errlen) {
  return no_throw([&] { return ua2a_impl_plan(in_slabs, out_slabs, B, S_local, H, D, w, mode,
                                              chunked, elem_bytes, forced_path, tuning, num_sms,
                                              out, err, errlen); });
}

int ulysses_a2a_get_settings(const ulysses_a2a_ctx* ctx, int32_t* path, ulysses_a2a_tuning_t* t) {
  return no_throw([&] { return ua2a_impl_get_settings(ctx, path, t); });
}

int ulysses_a2a_peer_create(ulysses_a2a_ctx* ctx, int rank, int world, size_t window_bytes,
                            ulysses_a2a_peer** out, void* handle_out) {
  return no_throw([&] { return ua2a_impl_peer_create(ctx, rank, world, window_bytes, out,
                                                     handle_out); });
}

int ulysses_a2a_peer_open(ulysses_a2a_peer* p, const void* handles) {
  return no_throw([&] { return ua2a_impl_peer_open(p, handles); });
}

int ulysses_a2a_peer_publish(ulysses_a2a_peer* p, const void* in_local, int64_t B, int64_t S_local,
                             int64_t H, int64_t D, int mode, int64_t row_pitch, void* stream) {
  return no_throw([&] { return ua2a_impl_peer_publish(p, in_local, B, S_local, H, D, mode,
                                                      row_pitch, stream); });
}

int ulysses_a2a_peer_pull(ulysses_a2a_peer* p, void* out_local, int64_t B, int64_t S_local,
                          int64_t H, int64_t D, int mode, int64_t row_pitch, void* stream) {
  return no_throw([&] { return ua2a_impl_peer_pull(p, out_local, B, S_local, H, D, mode, row_pitch,
                                                   stream); });
}

int ulysses_a2a_peer_close(ulysses_a2a_peer* p) {
  return no_throw([&] { return ua2a_impl_peer_close(p); });
}

int ulysses_a2a_peer_destroy(ulysses_a2a_peer* p) {
  return no_throw([&] { return ua2a_impl_peer_destroy(p); });
}

int ulysses_a2a_run_noalloc(const void* const* in_slabs, void* const* out_slabs, int64_t B,
                            int64_t S_local, int64_t H, int64_t D, int w, int mode, int chunked,
                            int elem_bytes, void* stream, int wait, char* err, size_t errlen) {
  return no_throw([&] { return ua2a_impl_run_noalloc(in_slabs, out_slabs, B, S_local, H, D, w, mode,
                                                     chunked, elem_bytes, stream, wait, err,
                                                     errlen); });
}

}  // extern "C"
