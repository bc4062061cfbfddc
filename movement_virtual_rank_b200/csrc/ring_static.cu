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
// cudaGetSymbolAddress and caches it.
#include <atomic>
#include <mutex>
#include <vector>

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
  void* scratch = nullptr;
  const int st0 = scratch_for_current_device(&scratch);
  if (st0 != COLL_OK) return st0;

  bool vec = true;
  for (int r = 0; r < nranks; ++r)
    vec = vec && (reinterpret_cast<uintptr_t>(send[r]) & 15) == 0 && (reinterpret_cast<uintptr_t>(recv[r]) & 15) == 0;
  const size_t g = 16 / es;
  const size_t seg = ((count + nranks - 1) / nranks + g - 1) / g * g;
  RingStepArgs a{};
  for (int r = 0; r < nranks; ++r) {
    a.in[r] = static_cast<const char*>(send[r]);
    a.out[r] = static_cast<char*>(recv[r]);
  }
  a.partial = static_cast<char*>(scratch);  // every partial is written before it is read: no clearing needed
  a.count = count;
  a.seg = seg;
  a.n = nranks;
  for (int k = 1; k < nranks; ++k) {
    a.k = k;
    const int st = launch_ring_rs_step(a, dtype, op, vec, s);
    if (st != COLL_OK) return st;
  }
  std::vector<CopyJob> jobs(nranks);
  for (int j = 1; j < nranks; ++j) {
    for (int c = 0; c < nranks; ++c) {
      const size_t lo = std::min(count, c * seg), hi = std::min(count, lo + seg);
      jobs[c] = {static_cast<const char*>(recv[(c + j - 1) % nranks]) + lo * es,
                 static_cast<char*>(recv[(c + j) % nranks]) + lo * es, (hi - lo) * es};
    }
    const int st = launch_copy_jobs(jobs.data(), nranks, s);
    if (st != COLL_OK) return st;
  }
  return COLL_OK;
}
