// ulysses_a2a.cu - C ABI of the B200 Ulysses 4D all-to-all re-layout: the
// context, the single-GPU entry points and every kernel launch.
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
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

using ua2a::StageParams;
using ua2a::TmaParams;
using ua2a::VecParams;

static_assert(ua2a::kVecResidentCtasPerSm == ua2a::kVecMinBlocksPerSm,
              "the planner's VEC residency must match the kernel's launch bound");


namespace ua2a {


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

// Vectors in flight per thread: 4, and 6 for the 8-byte mode-0 kernel, which
// holds them in its 32 registers (8 CTAs per SM) without spilling and so keeps
// as many bytes in flight per SM as the 16-byte kernel (200-byte runs, mode 0:
// 0.93 -> 0.96 of the copy bandwidth). Its mode-1 twin spills at 5.
template <typename V>
cudaError_t launch_vec_t(const VecParams& p, int mode, int grid, int block, cudaStream_t st) {
  constexpr int kU0 = sizeof(V) == 8 ? 6 : 4;
  return mode == 0 ? launch_pdl(ua2a::ua2a_vec_kernel<V, 0, kU0>, grid, block, 0, st, p)
                   : launch_pdl(ua2a::ua2a_vec_kernel<V, 1, 4>, grid, block, 0, st, p);
}

template <int MODE>
cudaError_t launch_shift_t(const VecParams& p, int grid, int block, cudaStream_t st) {
  switch (p.shift >> 2) {
    case 0: return launch_pdl(ua2a::ua2a_shift_kernel<MODE, 0>, grid, block, 0, st, p);
    case 1: return launch_pdl(ua2a::ua2a_shift_kernel<MODE, 1>, grid, block, 0, st, p);
    case 2: return launch_pdl(ua2a::ua2a_shift_kernel<MODE, 2>, grid, block, 0, st, p);
    default: return launch_pdl(ua2a::ua2a_shift_kernel<MODE, 3>, grid, block, 0, st, p);
  }
}

cudaError_t launch_vec(const VecParams& p, int vec_bytes, int peeled, int mode, int grid,
                       int block, cudaStream_t st) {
  if (peeled == 2)
    return mode == 0 ? launch_shift_t<0>(p, grid, block, st) : launch_shift_t<1>(p, grid, block, st);
  if (peeled)
    return mode == 0 ? launch_pdl(ua2a::ua2a_peel_kernel<0, UA2A_PEEL_ITEMS>, grid, block, 0, st, p)
                     : launch_pdl(ua2a::ua2a_peel_kernel<1, UA2A_PEEL_ITEMS>, grid, block, 0, st, p);
  switch (vec_bytes) {
    case 16: return launch_vec_t<uint4>(p, mode, grid, block, st);
    case 8: return launch_vec_t<uint2>(p, mode, grid, block, st);
    case 4: return launch_vec_t<unsigned int>(p, mode, grid, block, st);
    case 2: return launch_vec_t<unsigned short>(p, mode, grid, block, st);
    default: return launch_vec_t<unsigned char>(p, mode, grid, block, st);
  }
}

template <int G>
cudaError_t launch_stage_t(const StageParams& p, int mode, int grid, int block, size_t smem,
                           cudaStream_t st) {
  return mode == 0 ? launch_pdl(ua2a::ua2a_stage_kernel<G, 0>, grid, block, smem, st, p)
                   : launch_pdl(ua2a::ua2a_stage_kernel<G, 1>, grid, block, smem, st, p);
}

// The fixed-phase kernel's parameters from the staged kernel's: the same
// units and regions, plus the threads that move strided chunks and the rows
// between a thread's consecutive chunks.
PhaseParams phase_params(const StageParams& s) {
  PhaseParams p{};
  for (int k = 0; k < ULYSSES_A2A_MAX_W; ++k) {
    p.in[k] = s.in[k];
    p.out[k] = s.out[k];
  }
  p.S_local = s.S_local;
  p.b0 = s.b0;
  p.R = s.R;
  p.HDE = s.HDE;
  p.w = s.w;
  p.ng = s.ng;
  p.rows_per_tile = s.rows_per_tile;
  p.units = s.units;
  p.tile0 = s.tile0;
  p.RS = s.RS;
  p.Cg = s.Cg;
  p.nthr = (int32_t)ua2a::phase_movers(s.HDE);
  p.step_rows = 16 * p.nthr / s.HDE;
  p.div_T = s.div_T;
  p.div_w = s.div_w;
  p.div_R = s.div_R;
  p.div_HDE = ua2a::FastDiv((uint32_t)s.HDE);
  p.div_Cg = s.div_Cg;
  p.div_ng = ua2a::FastDiv((uint32_t)s.ng);
  // mode 0: gathered chunks c + m * Rp of a region share their phase (16 * Rp
  // is a multiple of R); regions padded to Cpad chunks, a multiple of Rp
  int64_t gr = 16;
  while (s.R % gr != 0) gr >>= 1;
  const int64_t Rp = s.R / gr;
  p.nthr0 = (int32_t)(Rp * (256 / Rp));
  p.Cpad = (int32_t)((s.Cg + Rp - 1) / Rp * Rp);
  p.div_Cpad = ua2a::FastDiv((uint32_t)p.Cpad);
  return p;
}

template <int G>
cudaError_t launch_phase_t(const PhaseParams& p, int mode, int grid, int block, size_t smem,
                           cudaStream_t st) {
  return mode == 0 ? launch_pdl(ua2a::ua2a_phase_kernel<G, 0>, grid, block, smem, st, p)
                   : launch_pdl(ua2a::ua2a_phase_kernel<G, 1>, grid, block, smem, st, p);
}

cudaError_t launch_stage(const StageParams& p, int piece_bytes, int fixed_phase, int mode, int grid,
                         int block, size_t smem, cudaStream_t st) {
  if (fixed_phase) {
    const PhaseParams q = phase_params(p);
    switch (piece_bytes) {
      case 8: return launch_phase_t<8>(q, mode, grid, block, smem, st);
      case 4: return launch_phase_t<4>(q, mode, grid, block, smem, st);
      case 2: return launch_phase_t<2>(q, mode, grid, block, smem, st);
      default: return launch_phase_t<1>(q, mode, grid, block, smem, st);
    }
  }
  switch (piece_bytes) {
    case 16: return launch_stage_t<16>(p, mode, grid, block, smem, st);
    case 8: return launch_stage_t<8>(p, mode, grid, block, smem, st);
    case 4: return launch_stage_t<4>(p, mode, grid, block, smem, st);
    case 2: return launch_stage_t<2>(p, mode, grid, block, smem, st);
    default: return launch_stage_t<1>(p, mode, grid, block, smem, st);
  }
}

template <int G>
cudaError_t stage_allow_t() {
  cudaError_t e = cudaFuncSetAttribute(ua2a::ua2a_stage_kernel<G, 0>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)ua2a::kStageSmemMax);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(ua2a::ua2a_stage_kernel<G, 1>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ua2a::kStageSmemMax);
  return e;
}

template <int G>
cudaError_t phase_allow_t() {
  cudaError_t e = cudaFuncSetAttribute(ua2a::ua2a_phase_kernel<G, 0>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)ua2a::kStageSmemMax);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(ua2a::ua2a_phase_kernel<G, 1>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ua2a::kStageSmemMax);
  return e;
}

cudaError_t stage_allow_max_smem() {
  cudaError_t e = phase_allow_t<8>();
  if (e == cudaSuccess) e = phase_allow_t<4>();
  if (e == cudaSuccess) e = phase_allow_t<2>();
  if (e == cudaSuccess) e = phase_allow_t<1>();
  if (e == cudaSuccess) e = stage_allow_t<16>();
  if (e == cudaSuccess) e = stage_allow_t<8>();
  if (e == cudaSuccess) e = stage_allow_t<4>();
  if (e == cudaSuccess) e = stage_allow_t<2>();
  if (e == cudaSuccess) e = stage_allow_t<1>();
  return e;
}

VecParams vec_params(const void* const* in, void* const* out, int nin, int nout, int64_t S, int w,
                     int E, const ulysses_a2a_plan_t& pl, int64_t units, int64_t nb, int64_t nt,
                     int nr, int nj, uint32_t r0, uint32_t r_stride, uint32_t j0, int64_t tile0) {
  VecParams p{};
  for (int k = 0; k < nin; ++k) p.in[k] = static_cast<const char*>(in[k]);
  for (int k = 0; k < nout; ++k) p.out[k] = static_cast<char*>(out[k]);
  p.S_local = S;
  p.srow = pl.row_pitch * E / pl.vec_bytes;
  if (pl.peeled) {
    // whole 16-byte destination vectors between each run's head and tail; the
    // source runs start `shift` bytes further past their boundary
    const int32_t a_in = (int32_t)(reinterpret_cast<uintptr_t>(in[0]) & 15u);
    const int32_t a_out = (int32_t)(reinterpret_cast<uintptr_t>(out[0]) & 15u);
    p.run = pl.row_bytes;
    p.nv = pl.row_bytes / 16 - (a_out ? 1 : 0);
    p.head = (16 - a_out) & 15;
    p.shift = (a_in - a_out) & 15;
  } else {
    p.nv = pl.row_bytes / pl.vec_bytes;
  }
  p.w = w;
  p.rows_per_tile = (int32_t)pl.rows_per_tile;
  p.units = (uint32_t)units;
  p.order = pl.order;
  p.tile0 = (uint32_t)tile0;
  p.r0 = r0;
  p.r_stride = r_stride;
  p.j0 = j0;
  p.div_T = ua2a::FastDiv((uint32_t)nt);
  p.div_nr = ua2a::FastDiv((uint32_t)nr);
  p.div_nj = ua2a::FastDiv((uint32_t)nj);
  p.div_nb = ua2a::FastDiv((uint32_t)nb);
  p.div_nv = ua2a::FastDiv((uint32_t)p.nv);
  return p;
}

StageParams stage_params(int64_t S, int w, int ntensors, int E, const ulysses_a2a_plan_t& pl,
                         int64_t nt, int64_t units) {
  StageParams p{};
  p.S_local = S;
  p.P = pl.row_pitch * E;
  p.R = (int32_t)pl.row_bytes;
  p.ng = w * ntensors;
  p.HDE = (int32_t)(pl.row_bytes * p.ng);
  p.w = w;
  p.rows_per_tile = (int32_t)pl.rows_per_tile;
  p.units = (uint32_t)units;
  StageGeometry sg;
  stage_geometry(pl.row_bytes, p.ng, S, (int)pl.rows_per_tile, &sg, pl.fixed_phase != 0);
  p.RS = (int32_t)sg.RS;
  p.Cs = (int32_t)sg.Cs;
  p.Cg = (int32_t)sg.Cg;
  p.div_T = ua2a::FastDiv((uint32_t)nt);
  p.div_w = ua2a::FastDiv((uint32_t)w);
  p.div_R = ua2a::FastDiv((uint32_t)p.R);
  p.div_ng = ua2a::FastDiv((uint32_t)p.ng);
  p.div_Cs = ua2a::FastDiv((uint32_t)p.Cs);
  p.div_Cg = ua2a::FastDiv((uint32_t)p.Cg);
  return p;
}

// run_device: see internal.h.
int run_device(ulysses_a2a_ctx* ctx, const void* const* in, void* const* out, int64_t B, int64_t S,
               int64_t H, int64_t D, int w, int mode, int chunked, cudaStream_t st,
               const ulysses_a2a_plan_t& pl, int64_t tile0, int64_t ntiles, int only_out,
               int ntensors) {
  const int64_t nb = chunked ? 1 : B;
  const int launches = chunked ? (int)B : 1;
  const int64_t nt = ntiles < 0 ? pl.tiles_per_block : ntiles;
  // a one-output launch covers rank only_out's head group of each tensor
  // (mode 0) or its sequence block j (mode 1)
  const int nr = (only_out >= 0 && mode == 0) ? ntensors : w * ntensors;
  const int nj = (only_out >= 0 && mode == 1) ? 1 : w;
  const bool staged = pl.path == ULYSSES_A2A_PATH_STAGED;
  // staged units cover every head group of their rows
  const int64_t units = staged ? (int64_t)nb * nj * nt : (int64_t)nr * nb * nj * nt;
  if (only_out >= 0 && pl.path != ULYSSES_A2A_PATH_VEC)
    return fail(ctx, ULYSSES_A2A_ERR_UNSUPPORTED, "one-output launches use the VEC path");
  if (ntensors > 1 && pl.path == ULYSSES_A2A_PATH_TMA)
    return fail(ctx, ULYSSES_A2A_ERR_UNSUPPORTED, "packed launches use the VEC or staged path");
  int grid = pl.grid;
  if (nt != pl.tiles_per_block) {
    if (pl.path == ULYSSES_A2A_PATH_TMA && pl.chunk_units > 0)
      grid = (int)((units + pl.chunk_units - 1) / pl.chunk_units);
    else if (units < grid)
      grid = (int)units;
  }
  if (staged) {
    StageParams p = stage_params(S, w, ntensors, ctx->elem_bytes, pl, nt, units);
    const int nin = mode == 0 ? w : w * ntensors;
    const int nout = mode == 0 ? w * ntensors : w;
    for (int k = 0; k < nin; ++k) p.in[k] = static_cast<const char*>(in[k]);
    for (int k = 0; k < nout; ++k) p.out[k] = static_cast<char*>(out[k]);
    p.tile0 = (uint32_t)tile0;
    if (!ctx->stage_smem_set) {
      cudaError_t e = stage_allow_max_smem();
      if (e != cudaSuccess) return cuda_fail(ctx, "cudaFuncSetAttribute (staged kernels)", e);
      ctx->stage_smem_set = true;
    }
    for (int l = 0; l < launches; ++l) {
      p.b0 = chunked ? l : 0;
      cudaError_t e = launch_stage(p, pl.vec_bytes, pl.fixed_phase, mode, grid, pl.block,
                                   (size_t)pl.smem_bytes, st);
      if (e != cudaSuccess) return cuda_fail(ctx, "staged kernel launch", e);
      ctx->launches++;
    }
    return ULYSSES_A2A_OK;
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
  const int nin = mode == 0 ? w : w * ntensors;
  const int nout = mode == 0 ? w * ntensors : w;
  VecParams p = vec_params(in, out, nin, nout, S, w, ctx->elem_bytes, pl, units, nb, nt, nr, nj,
                           (only_out >= 0 && mode == 0) ? (uint32_t)only_out : 0u,
                           (only_out >= 0 && mode == 0) ? (uint32_t)w : 1u,
                           (only_out >= 0 && mode == 1) ? (uint32_t)only_out : 0u, tile0);
  for (int l = 0; l < launches; ++l) {
    p.b0 = chunked ? l : 0;
    cudaError_t e = launch_vec(p, pl.vec_bytes, pl.peeled, mode, grid, pl.block, st);
    if (e != cudaSuccess) return cuda_fail(ctx, "VEC kernel launch", e);
    ctx->launches++;
  }
  return ULYSSES_A2A_OK;
}

int plan_for(ulysses_a2a_ctx* ctx, const void* const* in, void* const* out, int64_t B, int64_t S,
             int64_t H, int64_t D, int w, int mode, int chunked, ulysses_a2a_plan_t* pl,
             int64_t row_pitch, int ntensors) {
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
    else if (s == "staged") *path = ULYSSES_A2A_PATH_STAGED;
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

}  // namespace ua2a

namespace ua2a {

cudaError_t tma_allow_max_smem() {
  cudaError_t e = cudaFuncSetAttribute(ua2a_tma_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kTmaSmemMax);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(ua2a_tma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kTmaSmemMax);
  return e;
}

}  // namespace ua2a

using namespace ua2a;

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
  ua2a::ua2a_wait_selftest_kernel<0><<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      ctx->d_status, (uint64_t)limit_us * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(ctx, "self-test kernel launch", e);
  ctx->launches++;
  return ULYSSES_A2A_OK;
}

static int ua2a_impl_set_path(ulysses_a2a_ctx* ctx, int path) {
  if (ctx == nullptr) return ULYSSES_A2A_ERR_INVALID;
  if (path < ULYSSES_A2A_PATH_AUTO || path > ULYSSES_A2A_PATH_STAGED)
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
    t->staged_form = u.staged_form;
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

}  // extern "C"
