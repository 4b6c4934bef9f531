// peer.cu - the multi-GPU exchange of the Ulysses 4D all-to-all through
// published windows (ulysses_a2a_peer_* in include/ulysses_a2a.h).
#include <chrono>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <random>
#include <string>
#include <vector>

#include <unistd.h>

#include "internal.h"

using namespace ua2a;

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

// A byte offset into the windows: a multiple of the element size, inside them.
static int check_window_offset(ulysses_a2a_peer* p, size_t window_offset, const char* who) {
  if (window_offset % (size_t)p->ctx->elem_bytes != 0 || window_offset > p->window_bytes)
    return fail(p->ctx, ULYSSES_A2A_ERR_INVALID,
                std::string(who) + ": window_offset must be a multiple of the element size "
                                   "inside the window");
  return ULYSSES_A2A_OK;
}

static int ua2a_impl_peer_publish(ulysses_a2a_peer* p, const void* in_local, int64_t B,
                                  int64_t S_local, int64_t H, int64_t D, int mode,
                                  int64_t row_pitch, size_t window_offset, void* stream) {
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
  int rc = check_window_offset(p, window_offset, "peer_publish");
  if (rc) return rc;
  const size_t room = p->window_bytes - window_offset;
  void* dst = static_cast<char*>(p->own) + window_offset;
  // the copy, as a one-rank re-layout: mode 0 keeps [B, S, H, D] (dropping the
  // pitch); mode 1 copies [B, S*w, H/w, D]
  const int64_t S1 = mode == 0 ? S_local : S_local * w;
  const int64_t H1 = mode == 0 ? H : H / w;
  if (in_local == dst && (row_pitch == 0 || row_pitch == H1 * D)) {
    // the slab was written into the window in place: nothing to copy
    int64_t bytes = 0;
    if (ua2a::mul_overflows(B, S1, &bytes) || ua2a::mul_overflows(bytes, H1, &bytes) ||
        ua2a::mul_overflows(bytes, D, &bytes) ||
        ua2a::mul_overflows(bytes, (int64_t)ctx->elem_bytes, &bytes) || (uint64_t)bytes > room)
      return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_publish: the slab exceeds the window");
    return ULYSSES_A2A_OK;
  }
  const void* in[1] = {in_local};
  void* out[1] = {dst};
  ulysses_a2a_plan_t pl;
  rc = plan_for(ctx, in, out, B, S1, H1, D, 1, 0, 0, &pl, row_pitch);
  if (rc) return rc;
  if (pl.units == 0) return ULYSSES_A2A_OK;
  if ((uint64_t)pl.payload_bytes > room)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_publish: the slab (" + std::to_string(pl.payload_bytes) +
                                                  " bytes) exceeds the window (" + std::to_string(room) +
                                                  " bytes from the offset)");
  DeviceGuard g(ctx->device);
  if (!g.ok) return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "cannot select the context's device");
  const int64_t in_bytes = ((B * S1 - 1) * pl.row_pitch + H1 * D) * (int64_t)ctx->elem_bytes;
  rc = check_residency(ctx, in, 1, in_bytes, "input");
  if (rc) return rc;
  return run_device(ctx, in, out, B, S1, H1, D, 1, 0, 0, static_cast<cudaStream_t>(stream), pl);
}

static int ua2a_impl_peer_pull(ulysses_a2a_peer* p, void* out_local, int64_t B, int64_t S_local,
                               int64_t H, int64_t D, int mode, int64_t row_pitch,
                               size_t window_offset, void* stream) {
  if (p == nullptr) return ULYSSES_A2A_ERR_INVALID;
  ulysses_a2a_ctx* ctx = p->ctx;
  ctx->last_error.clear();
  if (!p->open) return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_pull: the peer windows are not open");
  const int w = p->world;
  int rc = check_window_offset(p, window_offset, "peer_pull");
  if (rc) return rc;
  // every rank's window, read from the offset on
  std::vector<const void*> ins(w);
  for (int k = 0; k < w; ++k) ins[k] = static_cast<const char*>(p->bases[k]) + window_offset;
  std::vector<void*> outs(w, nullptr);
  outs[p->rank] = out_local;
  std::string err;
  ulysses_a2a_plan_t pl;
  // row_pitch belongs to the [B, S, H, D] side: the windows in mode 0, the output in mode 1
  rc = ua2a::make_plan(ins.data(), outs.data(), B, S_local, H, D, w, mode, 0, ctx->elem_bytes,
                       ULYSSES_A2A_PATH_VEC, ctx->tuning, ctx->num_sms, &pl, &err, row_pitch, p->rank);
  if (rc) return fail(ctx, rc, "peer_pull: " + err);
  if (pl.units == 0) return ULYSSES_A2A_OK;
  const int64_t strided_bytes = ((B * S_local - 1) * pl.row_pitch + H * D) * (int64_t)ctx->elem_bytes;
  const int64_t window_side = mode == 0 ? strided_bytes : pl.payload_bytes;
  if ((uint64_t)window_side > (uint64_t)(p->window_bytes - window_offset))
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_pull: the slab (" + std::to_string(window_side) +
                                                  " bytes) exceeds the windows (" +
                                                  std::to_string(p->window_bytes - window_offset) +
                                                  " bytes from the offset)");
  DeviceGuard g(ctx->device);
  if (!g.ok) return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "cannot select the context's device");
  const int64_t out_bytes = mode == 0 ? pl.payload_bytes : strided_bytes;
  const void* o[1] = {out_local};
  rc = check_residency(ctx, o, 1, out_bytes, "output");
  if (rc) return rc;
  return run_device(ctx, ins.data(), outs.data(), B, S_local, H, D, w, mode, 0,
                    static_cast<cudaStream_t>(stream), pl, 0, -1, p->rank);
}

static int ua2a_impl_peer_pull_packed(ulysses_a2a_peer* p, void* const* out_local, int ntensors,
                                      int64_t B, int64_t S_local, int64_t H, int64_t D, int mode,
                                      size_t window_offset, void* stream) {
  if (p == nullptr) return ULYSSES_A2A_ERR_INVALID;
  ulysses_a2a_ctx* ctx = p->ctx;
  ctx->last_error.clear();
  if (!p->open) return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_pull_packed: the peer windows are not open");
  const int w = p->world;
  const int T = ntensors;
  if (out_local == nullptr || T < 1 || (int64_t)T * w > ULYSSES_A2A_MAX_W)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID,
                "peer_pull_packed: need an output array and 1 <= ntensors, ntensors * world <= 64");
  if (mode != 0 && mode != 1) return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_pull_packed: mode must be 0 or 1");
  if (B < 0 || S_local < 0 || H < 0 || D < 0)
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_pull_packed: sizes must be >= 0");
  int rc = check_window_offset(p, window_offset, "peer_pull_packed");
  if (rc) return rc;
  int64_t slab = 0;  // one tensor's slab of one rank, either layout
  if (ua2a::mul_overflows(B, S_local, &slab) || ua2a::mul_overflows(slab, H, &slab) ||
      ua2a::mul_overflows(slab, D, &slab) || ua2a::mul_overflows(slab, (int64_t)ctx->elem_bytes, &slab) ||
      slab > (int64_t(1) << 56))
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_pull_packed: slab sizes overflow");
  // Mode 0: every window holds a packed [B, S, T, H, D] slab (rows of T*H*D
  // elements), tensor t's heads at element t*H*D of each row; this rank's
  // output slab of tensor t is out[t*w + rank]. Mode 1: every window holds T
  // dense [B, S*w, H/w, D] slabs, tensor t at byte t*slab, i.e. input slab
  // t*w + r of the packed launch; this rank's packed output is out[rank].
  std::vector<const void*> ins(mode == 0 ? w : (size_t)T * w);
  std::vector<void*> outs(mode == 0 ? (size_t)T * w : w, nullptr);
  for (int k = 0; k < w; ++k) {
    const char* base = static_cast<const char*>(p->bases[k]) + window_offset;
    if (mode == 0)
      ins[k] = base;
    else
      for (int t = 0; t < T; ++t) ins[(size_t)t * w + k] = base + (size_t)t * (size_t)slab;
  }
  if (mode == 0)
    for (int t = 0; t < T; ++t) outs[(size_t)t * w + p->rank] = out_local[t];
  else
    outs[p->rank] = out_local[0];
  std::string err;
  ulysses_a2a_plan_t pl;
  rc = ua2a::make_plan(ins.data(), outs.data(), B, S_local, H, D, w, mode, 0, ctx->elem_bytes,
                       ULYSSES_A2A_PATH_VEC, ctx->tuning, ctx->num_sms, &pl, &err, 0, p->rank, T);
  if (rc) return fail(ctx, rc, "peer_pull_packed: " + err);
  if (pl.units == 0) return ULYSSES_A2A_OK;
  if ((uint64_t)slab * (uint64_t)T > (uint64_t)(p->window_bytes - window_offset))
    return fail(ctx, ULYSSES_A2A_ERR_INVALID, "peer_pull_packed: the " + std::to_string(T) +
                                                  " slabs exceed the windows from the offset");
  DeviceGuard g(ctx->device);
  if (!g.ok) return fail(ctx, ULYSSES_A2A_ERR_DEVICE, "cannot select the context's device");
  if (mode == 0) {
    std::vector<const void*> o(out_local, out_local + T);
    rc = check_residency(ctx, o.data(), T, slab, "output");
  } else {
    const void* o[1] = {out_local[0]};
    rc = check_residency(ctx, o, 1, slab * T, "output");
  }
  if (rc) return rc;
  return run_device(ctx, ins.data(), outs.data(), B, S_local, H, D, w, mode, 0,
                    static_cast<cudaStream_t>(stream), pl, 0, -1, p->rank, T);
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

extern "C" {

int ulysses_a2a_peer_create(ulysses_a2a_ctx* ctx, int rank, int world, size_t window_bytes,
                            ulysses_a2a_peer** out, void* handle_out) {
  return no_throw([&] { return ua2a_impl_peer_create(ctx, rank, world, window_bytes, out,
                                                     handle_out); });
}

int ulysses_a2a_peer_open(ulysses_a2a_peer* p, const void* handles) {
  return no_throw([&] { return ua2a_impl_peer_open(p, handles); });
}

int ulysses_a2a_peer_publish(ulysses_a2a_peer* p, const void* in_local, int64_t B, int64_t S_local,
                             int64_t H, int64_t D, int mode, int64_t row_pitch,
                             size_t window_offset, void* stream) {
  return no_throw([&] {
    return ua2a_impl_peer_publish(p, in_local, B, S_local, H, D, mode, row_pitch, window_offset,
                                  stream);
  });
}

int ulysses_a2a_peer_pull(ulysses_a2a_peer* p, void* out_local, int64_t B, int64_t S_local,
                          int64_t H, int64_t D, int mode, int64_t row_pitch, size_t window_offset,
                          void* stream) {
  return no_throw([&] {
    return ua2a_impl_peer_pull(p, out_local, B, S_local, H, D, mode, row_pitch, window_offset,
                               stream);
  });
}

int ulysses_a2a_peer_pull_packed(ulysses_a2a_peer* peer, void* const* out_local, int ntensors,
                                 int64_t B, int64_t S_local, int64_t H, int64_t D, int mode,
                                 size_t window_offset, void* stream) {
  return no_throw([&] { return ua2a_impl_peer_pull_packed(peer, out_local, ntensors, B, S_local, H, D,
                                                          mode, window_offset, stream); });
}

int ulysses_a2a_peer_close(ulysses_a2a_peer* p) {
  return no_throw([&] { return ua2a_impl_peer_close(p); });
}

int ulysses_a2a_peer_destroy(ulysses_a2a_peer* p) {
  return no_throw([&] { return ua2a_impl_peer_destroy(p); });
}

}  // extern "C"
