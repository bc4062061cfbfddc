// coll_all_reduce_ring_noalloc: the ring all-reduce with its scratch in a
// fixed device array compiled into this library, for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is not available or not
// allowed -- a plugin handed only the caller's buffers, a hook running inside
// another framework's memory pool, a process whose allocations are capped or
// frozen after start-up.  coll_all_reduce(RING) needs a caller-provided
// workspace for the partial sums that travel round the ring; this entry point
// takes no workspace and never allocates: the partials live in g_ring_scratch
// below, a file-scope __device__ array that every GPU loading the library
// holds until the process exits.
//
// Host code cannot use g_ring_scratch's name as an address (on the host it
// names a stand-in object, not device memory), so the first call on each
// device, with that device current, looks up the array's device address with
// cudaGetSymbolAddress and caches it.  Under lazy module loading (the CUDA
// default) that lookup is also when the driver places the array on the
// device, so it is done before any shortcut: a call with count == 0 is the
// warm-up a caller makes before reserving the rest of the device's memory.
#include <atomic>
#include <mutex>

#include "coll.h"
#include "common.cuh"
#include "internal.h"

namespace mvr {

static __device__ __align__(256) unsigned char g_ring_scratch[COLL_RING_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_setup_mu;
std::atomic<void*> g_scratch_ptr[COLL_MAX_RANKS];  // per device ordinal

// device address of g_ring_scratch on the current device (looked up once)
int scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_status(e);
  if (dev < 0 || dev >= COLL_MAX_RANKS) return COLL_ERR_UNSUPPORTED;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
      e = cudaGetSymbolAddress(&p, g_ring_scratch);
      if (e != cudaSuccess || p == nullptr) return launch_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return COLL_OK;
}

inline bool overlap(const void* a, size_t an, const void* b, size_t bn) {
  if (an == 0 || bn == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + bn && y < x + an;
}

}  // namespace
}  // namespace mvr

using namespace mvr;

extern "C" int coll_all_reduce_ring_noalloc(const void* const* send, void* const* recv, int nranks, size_t count,
                                            coll_dtype_t dtype, coll_op_t op, coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es || op < COLL_SUM || op > COLL_PROD) return COLL_ERR_UNSUPPORTED;
  if (nranks < 1 || nranks > COLL_MAX_RANKS || send == nullptr || recv == nullptr) return COLL_ERR_INVALID_ARG;
  for (int r = 0; r < nranks; ++r)
    if (send[r] == nullptr || recv[r] == nullptr) return COLL_ERR_INVALID_ARG;
  // The address comes first, before the count == 0 and N == 1 shortcuts: the
  // first call on a device is where the driver places the array (under lazy
  // module loading, the default, that is when this file's module is loaded),
  // so a call with count == 0 serves as a warm-up that a caller can make
  // before it reserves the rest of the device's memory.
  void* scratch = nullptr;
  const int st0 = scratch_for_current_device(&scratch);
  if (st0 != COLL_OK) return st0;
  const size_t bytes = count * es;
  if (bytes == 0) return COLL_OK;
  if (count > COLL_RING_NOALLOC_MAX_COUNT) return COLL_ERR_WORKSPACE;  // beyond the fixed scratch
  for (int q = 0; q < nranks; ++q)
    for (int r = 0; r < nranks; ++r) {
      if (q < r && overlap(recv[q], bytes, recv[r], bytes)) return COLL_ERR_ALIAS;
      if (overlap(recv[q], bytes, send[r], bytes) && !(q == r && recv[q] == send[r])) return COLL_ERR_ALIAS;
    }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (nranks == 1) {
    if (send[0] == recv[0]) return COLL_OK;
    CopyJob j{static_cast<const char*>(send[0]), static_cast<char*>(recv[0]), bytes};
    return launch_copy_jobs(&j, 1, s);
  }
  bool vec = true;
  const char* in[COLL_MAX_RANKS];
  char* out[COLL_MAX_RANKS];
  for (int r = 0; r < nranks; ++r) {
    in[r] = static_cast<const char*>(send[r]);
    out[r] = static_cast<char*>(recv[r]);
    vec = vec && (reinterpret_cast<uintptr_t>(send[r]) & 15) == 0 && (reinterpret_cast<uintptr_t>(recv[r]) & 15) == 0;
  }
  // the same launches as coll_all_reduce(RING_STEPS); every partial is
  // written before it is read, so the array needs no clearing
  return launch_ring_steps(in, out, nranks, count, dtype, op, static_cast<char*>(scratch), vec, s);
}
