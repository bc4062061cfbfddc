// The extern "C" entry points of include/coll.h: argument validation, the
// overlap rules, the N == 1 and count == 0 shortcuts, and the choice of
// kernel.  No entry point allocates memory or synchronises the stream.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <cstdio>
#include <cstring>
#include <vector>

#include "coll.h"
#include "internal.h"

namespace mvr {

// per-dtype launchers defined in reduce_<dtype>.cu
int launch_reduce_bf16(const ReduceArgs&, coll_op_t, int, bool, int, cudaStream_t);
int launch_reduce_fp16(const ReduceArgs&, coll_op_t, int, bool, int, cudaStream_t);
int launch_reduce_fp32(const ReduceArgs&, coll_op_t, int, bool, int, cudaStream_t);
int launch_reduce_int32(const ReduceArgs&, coll_op_t, int, bool, int, cudaStream_t);
int launch_ring_bf16(const RingStepArgs&, coll_op_t, bool, cudaStream_t);
int launch_ring_fp16(const RingStepArgs&, coll_op_t, bool, cudaStream_t);
int launch_ring_fp32(const RingStepArgs&, coll_op_t, bool, cudaStream_t);
int launch_ring_int32(const RingStepArgs&, coll_op_t, bool, cudaStream_t);

enum { kAll = 0, kBlock = 1, kSame = 2, kOneShot = 3 };  // mirrors ReduceMode

static thread_local char g_cuda_msg[256];

int launch_status(cudaError_t e) {
  if (e == cudaSuccess) return COLL_OK;
  std::snprintf(g_cuda_msg, sizeof(g_cuda_msg), "CUDA error %d: %s", static_cast<int>(e), cudaGetErrorString(e));
  return COLL_ERR_CUDA;
}

int allow_dynamic_smem(const void* fn, size_t bytes, int* done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= COLL_MAX_RANKS) dev = 0;
  if (done[dev] >= static_cast<int>(bytes)) return COLL_OK;
  const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) {
    (void)cudaGetLastError();  // reported here; keep it from surfacing in a later call
    return launch_status(e);
  }
  done[dev] = static_cast<int>(bytes);
  return COLL_OK;
}

int num_sms() {
  static std::atomic<int> cache[COLL_MAX_RANKS];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= COLL_MAX_RANKS) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

// CTAs of `fn` that fit on the whole GPU at once (occupancy API), cached per
// kernel and device: the grid of a kernel that walks its data with a resident
// grid (the one-shot all-reduce, whose N readers of a tile must run together
// for L2 to serve the repeats).  A larger grid would run its extra CTAs as a
// short second wave after the first had finished its share.
int resident_ctas(const void* fn, int threads, size_t smem) {
  struct Entry {
    const void* fn;
    int dev, threads, per_sm;
  };
  static Entry table[256];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
      if (table[i].fn == fn && table[i].dev == dev && table[i].threads == threads) return table[i].per_sm * num_sms();
  }
  int v = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, fn, threads, smem) != cudaSuccess || v <= 0) {
    (void)cudaGetLastError();
    return num_sms() * 8;  // the grids' own cap; the launch reports any real error
  }
  std::lock_guard<std::mutex> lock(mu);
  if (used < 256) table[used++] = Entry{fn, dev, threads, v};
  return v * num_sms();
}

// Grids of the other streaming element kernels: one work item per thread, the
// CTAs launched in order and retired as they finish, rather than a resident
// grid walking the data with a stride.  Measured on B200: the two-shot
// all-reduce at 2 x 1 GiB 750 -> 650 us, at 8 x 256 MiB 707 -> 655 us, the LL
// packetised all-reduce at 8 x 256 MiB 1418 -> 1271 us, reduce_scatter at
// 8 x 128 MiB 176 -> 174 us.  The kernels keep their grid-stride loops, so a
// message larger than the grid still finishes.
uint64_t stream_grid(uint64_t units, int threads) {
  uint64_t g = (units + static_cast<uint64_t>(threads) - 1) / static_cast<uint64_t>(threads);
  if (g > kMaxStreamGrid) g = kMaxStreamGrid;
  return g < 1 ? 1 : g;
}

int elem_size(coll_dtype_t dt) {
  switch (dt) {
    case COLL_BF16:
    case COLL_FP16: return 2;
    case COLL_FP32:
    case COLL_INT32: return 4;
  }
  return 0;
}

int launch_reduce(const ReduceArgs& a, coll_dtype_t dt, coll_op_t op, int mode, bool vec, int bps, cudaStream_t s) {
  switch (dt) {
    case COLL_BF16: return launch_reduce_bf16(a, op, mode, vec, bps, s);
    case COLL_FP16: return launch_reduce_fp16(a, op, mode, vec, bps, s);
    case COLL_FP32: return launch_reduce_fp32(a, op, mode, vec, bps, s);
    case COLL_INT32: return launch_reduce_int32(a, op, mode, vec, bps, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

int launch_ring_rs_step(const RingStepArgs& a, coll_dtype_t dt, coll_op_t op, bool vec, cudaStream_t s) {
  switch (dt) {
    case COLL_BF16: return launch_ring_bf16(a, op, vec, s);
    case COLL_FP16: return launch_ring_fp16(a, op, vec, s);
    case COLL_FP32: return launch_ring_fp32(a, op, vec, s);
    case COLL_INT32: return launch_ring_int32(a, op, vec, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

int launch_ring_steps(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                      char* partial, bool vec, cudaStream_t s) {
  const int es = elem_size(dt);
  const size_t g = 16 / es;
  const size_t seg = ((count + n - 1) / n + g - 1) / g * g;
  RingStepArgs a{};
  for (int r = 0; r < n; ++r) {
    a.in[r] = in[r];
    a.out[r] = out[r];
  }
  a.partial = partial;
  a.count = count;
  a.seg = seg;
  a.n = n;
  for (int k = 1; k < n; ++k) {  // reduce-scatter phase
    a.k = k;
    const int st = launch_ring_rs_step(a, dt, op, vec, s);
    if (st != COLL_OK) return st;
  }
  std::vector<CopyJob> jobs(n);
  for (int j = 1; j < n; ++j) {  // all-gather phase: rank c+j copies chunk c from rank c+j-1
    for (int c = 0; c < n; ++c) {
      const size_t lo = std::min(count, c * seg), hi = std::min(count, lo + seg);
      jobs[c] = {out[(c + j - 1) % n] + lo * es, out[(c + j) % n] + lo * es, (hi - lo) * es};
    }
    const int st = launch_copy_jobs(jobs.data(), n, s);
    if (st != COLL_OK) return st;
  }
  return COLL_OK;
}

}  // namespace mvr

using namespace mvr;

namespace {

inline cudaStream_t S(coll_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }
inline uintptr_t U(const void* p) { return reinterpret_cast<uintptr_t>(p); }
inline bool al16(const void* p) { return (U(p) & 15) == 0; }

// [a, a+an) and [b, b+bn) share a byte
inline bool overlap(const void* a, size_t an, const void* b, size_t bn) {
  if (an == 0 || bn == 0) return false;
  return U(a) < U(b) + bn && U(b) < U(a) + an;
}

inline bool valid_n(int n) { return n >= 1 && n <= COLL_MAX_RANKS; }
inline bool valid_op(coll_op_t op) { return op >= COLL_SUM && op <= COLL_PROD; }

template <typename P>
bool all_nonnull(P const* p, int n) {
  if (p == nullptr) return false;
  for (int i = 0; i < n; ++i)
    if (p[i] == nullptr) return false;
  return true;
}

// outputs pairwise disjoint
bool outputs_disjoint(void* const* out, int n, size_t bytes) {
  for (int i = 0; i < n; ++i)
    for (int j = i + 1; j < n; ++j)
      if (overlap(out[i], bytes, out[j], bytes)) return false;
  return true;
}

size_t seg_elems(size_t count, int n, int es) {
  const size_t g = 16 / es;
  const size_t per = (count + n - 1) / n;
  return (per + g - 1) / g * g;
}

int blocks_per_slice(uint64_t slice_units, int nslices) {
  const uint64_t cap = std::max<uint64_t>(1, kMaxStreamGrid / static_cast<uint64_t>(nslices));
  return static_cast<int>(std::min(stream_grid(slice_units, kBlockThreads), cap));
}

int copy_one(const void* src, void* dst, size_t bytes, cudaStream_t s) {
  if (src == dst || bytes == 0) return COLL_OK;
  CopyJob j{static_cast<const char*>(src), static_cast<char*>(dst), bytes};
  return launch_copy_jobs(&j, 1, s);
}

size_t ring_ws(size_t count) { return (count * 4 + 255) / 256 * 256; }

}  // namespace

extern "C" {

int coll_version(void) { return 10000; }

const char* coll_strerror(int status) {
  switch (status) {
    case COLL_OK: return "ok";
    case COLL_ERR_INVALID_ARG: return "invalid argument";
    case COLL_ERR_UNSUPPORTED: return "unsupported dtype / op / algorithm";
    case COLL_ERR_ALIAS: return "buffers overlap in a way this collective does not allow";
    case COLL_ERR_CUDA: return g_cuda_msg[0] ? g_cuda_msg : "CUDA error";
    case COLL_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
  }
  return "unknown status";
}

// ------------------------------------------------------------- Broadcast ----
int coll_broadcast(void* const* bufs, int nranks, size_t count, coll_dtype_t dtype, int src, coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || src < 0 || src >= nranks || !all_nonnull(bufs, nranks)) return COLL_ERR_INVALID_ARG;
  const size_t bytes = count * es;
  if (bytes == 0 || nranks == 1) return COLL_OK;
  if (!outputs_disjoint(bufs, nranks, bytes)) return COLL_ERR_ALIAS;
  FanoutArgs a{};
  a.src[0] = static_cast<const char*>(bufs[src]);
  a.ns = 1;
  for (int q = 0; q < nranks; ++q)
    if (q != src) a.dst[a.nd++] = static_cast<char*>(bufs[q]);
  a.bytes = bytes;
  a.dst_stride = 0;
  return launch_fanout(a, S(stream));
}

// ---------------------------------------------------------------- Gather ----
int coll_gather(const void* const* send, void* recv_dst, int nranks, size_t rows, size_t cols_per_rank,
                coll_dtype_t dtype, int dst, coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || dst < 0 || dst >= nranks || !all_nonnull(send, nranks) || recv_dst == nullptr || rows == 0)
    return COLL_ERR_INVALID_ARG;
  const size_t blk = rows * cols_per_rank * es;  // one rank's block
  if (blk == 0) return COLL_OK;
  const size_t total = blk * nranks;
  char* out = static_cast<char*>(recv_dst);
  for (int r = 0; r < nranks; ++r) {
    if (!overlap(send[r], blk, out, total)) continue;
    const bool in_place = rows == 1 && r == dst && send[r] == out + static_cast<size_t>(r) * blk;
    if (!in_place) return COLL_ERR_ALIAS;
  }
  if (rows == 1) {
    std::vector<CopyJob> jobs;
    for (int r = 0; r < nranks; ++r) {
      char* d = out + static_cast<size_t>(r) * blk;
      if (send[r] != d) jobs.push_back({static_cast<const char*>(send[r]), d, blk});
    }
    return launch_copy_jobs(jobs.data(), static_cast<int>(jobs.size()), S(stream));
  }
  GatherRowsArgs a{};
  for (int r = 0; r < nranks; ++r) a.src[r] = static_cast<const char*>(send[r]);
  a.dst = out;
  a.rows = rows;
  a.row_bytes = cols_per_rank * es;
  a.dst_pitch = a.row_bytes * nranks;
  a.n = nranks;
  return launch_gather_rows(a, S(stream));
}

// ---------------------------------------------------------------- Reduce ----
int coll_reduce(const void* const* send, void* recv_dst, int nranks, size_t count, coll_dtype_t dtype, coll_op_t op,
                int dst, coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!valid_op(op)) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || dst < 0 || dst >= nranks || !all_nonnull(send, nranks) || recv_dst == nullptr)
    return COLL_ERR_INVALID_ARG;
  const size_t bytes = count * es;
  if (bytes == 0) return COLL_OK;
  for (int r = 0; r < nranks; ++r)
    if (overlap(send[r], bytes, recv_dst, bytes) && !(r == dst && send[r] == recv_dst)) return COLL_ERR_ALIAS;
  if (nranks == 1) return copy_one(send[0], recv_dst, bytes, S(stream));
  ReduceArgs a{};
  bool vec = al16(recv_dst);
  for (int r = 0; r < nranks; ++r) {
    a.in[r] = static_cast<const char*>(send[r]);
    vec = vec && al16(send[r]);
  }
  a.out[0] = static_cast<char*>(recv_dst);
  a.count = count;
  a.seg = count;
  a.nin = nranks;
  a.nout = 1;
  a.nslices = 1;
  const int bps = blocks_per_slice(vec ? count * es / 16 : count, 1);
  return launch_reduce(a, dtype, op, kSame, vec, bps, S(stream));
}

// --------------------------------------------------------------- Scatter ----
int coll_scatter(const void* send_src, void* const* recv, int nranks, size_t count_per_rank, coll_dtype_t dtype,
                 int src, coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || src < 0 || src >= nranks || send_src == nullptr || !all_nonnull(recv, nranks))
    return COLL_ERR_INVALID_ARG;
  const size_t blk = count_per_rank * es;
  if (blk == 0) return COLL_OK;
  const char* in = static_cast<const char*>(send_src);
  if (!outputs_disjoint(recv, nranks, blk)) return COLL_ERR_ALIAS;
  std::vector<CopyJob> jobs;
  for (int r = 0; r < nranks; ++r) {
    const char* sp = in + static_cast<size_t>(r) * blk;
    if (overlap(recv[r], blk, in, blk * nranks)) {
      if (!(r == src && recv[r] == sp)) return COLL_ERR_ALIAS;
      continue;  // already in place
    }
    jobs.push_back({sp, static_cast<char*>(recv[r]), blk});
  }
  return launch_copy_jobs(jobs.data(), static_cast<int>(jobs.size()), S(stream));
}

// --------------------------------------------------------- ReduceScatter ----
int coll_reduce_scatter(const void* const* send, void* const* recv, int nranks, size_t recv_count,
                        coll_dtype_t dtype, coll_op_t op, coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!valid_op(op)) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || !all_nonnull(send, nranks) || !all_nonnull(recv, nranks)) return COLL_ERR_INVALID_ARG;
  const size_t blk = recv_count * es;
  if (blk == 0) return COLL_OK;
  const size_t in_bytes = blk * nranks;
  if (!outputs_disjoint(recv, nranks, blk)) return COLL_ERR_ALIAS;
  for (int q = 0; q < nranks; ++q)
    for (int r = 0; r < nranks; ++r)
      if (overlap(recv[q], blk, send[r], in_bytes) &&
          !(q == r && recv[q] == static_cast<const char*>(send[r]) + static_cast<size_t>(q) * blk))
        return COLL_ERR_ALIAS;
  if (nranks == 1) return copy_one(send[0], recv[0], blk, S(stream));
  ReduceArgs a{};
  bool vec = (blk % 16) == 0;
  for (int r = 0; r < nranks; ++r) {
    a.in[r] = static_cast<const char*>(send[r]);
    a.out[r] = static_cast<char*>(recv[r]);
    vec = vec && al16(send[r]) && al16(recv[r]);
  }
  a.count = recv_count * nranks;
  a.seg = recv_count;
  a.nin = nranks;
  a.nout = 1;
  a.nslices = nranks;
  const int bps = blocks_per_slice(vec ? blk / 16 : recv_count, nranks);
  return launch_reduce(a, dtype, op, kBlock, vec, bps, S(stream));
}

// ------------------------------------------------------------- AllReduce ----
// RING runs as the one-launch ring measured fastest on B200 for the rank
// count and the bytes per rank (cold inputs, 1 KiB .. 256 MiB per rank at 2,
// 3, 4 and 8 virtual ranks), when the buffers allow one: the ranks as lanes
// of a warp (RING_LANE) at 2 ranks, at 3 and 4 ranks up to 256 KiB and at 5
// and more up to 16 KiB; above those, where RING_LANE's per-rank 64-byte
// accesses load the L1 data pipe, the ranks as warps of a CTA (RING_CTA).
// The cluster form and the stream-ordered steps were slower at every size.
// Every form gives the same bits.
static coll_algo_t ring_form(int nranks, size_t bytes, bool vec) {
  if (!vec || !ring_cta_supported(nranks)) return COLL_ALGO_RING_STEPS;
  if (nranks == 2 || (nranks <= 4 && bytes <= (256u << 10)) || bytes <= (16u << 10)) return COLL_ALGO_RING_LANE;
  return COLL_ALGO_RING_CTA;
}

// AUTO: the form measured fastest on B200 for the rank count and the bytes
// per rank (cold inputs, 1 KiB .. 256 MiB per rank, 2, 3, 4 and 8 virtual
// ranks, every one-launch form).  At 3 and 4 ranks the one-shot, every output
// rank reading all inputs itself, beats the owner segments on small messages
// (by up to 0.3 us); everywhere else the two-shot is fastest or tied (at 8
// ranks and 256 MiB the CTA ring is within 1.5% of it).  Rank counts that were
// not measured take the nearest measured rule: 5 and more the 8-rank one.
// The one-shot cannot run in place, so an in-place call takes the two-shot.
static coll_algo_t auto_form(int nranks, size_t bytes, bool in_place) {
  if (in_place) return COLL_ALGO_TWOSHOT;
  if (nranks == 3 && bytes <= (256u << 10)) return COLL_ALGO_ONESHOT;
  if (nranks == 4 && bytes <= (64u << 10)) return COLL_ALGO_ONESHOT;
  return COLL_ALGO_TWOSHOT;
}

size_t coll_all_reduce_workspace_size(int nranks, size_t count, coll_dtype_t dtype, coll_algo_t algo) {
  if (!valid_n(nranks) || !elem_size(dtype)) return 0;
  // 256-byte header (status pair at bytes 16..23), then the fp32 / int32 partials
  if (algo == COLL_ALGO_RING || algo == COLL_ALGO_RING_STEPS) return 256 + ring_ws(count);
  if (algo == COLL_ALGO_RING_LL) return std::max(ring_ll_workspace(nranks, count, elem_size(dtype)), 256 + ring_ws(count));
  if (algo == COLL_ALGO_TWOSHOT_LL) return twoshot_ll_workspace(nranks, count, elem_size(dtype));
  if (algo == COLL_ALGO_TWOSHOT_LL128) return twoshot_ll128_workspace(nranks, count, elem_size(dtype));
  return 0;
}

int coll_all_reduce_form(int nranks, size_t count, coll_dtype_t dtype, coll_algo_t algo, int aligned) {
  const int es = elem_size(dtype);
  if (!es || !valid_n(nranks)) return COLL_ERR_INVALID_ARG;
  if (algo < COLL_ALGO_AUTO || algo > COLL_ALGO_RING_WIRE) return COLL_ERR_UNSUPPORTED;
  const bool vec = aligned != 0;
  switch (algo) {
    case COLL_ALGO_AUTO: return auto_form(nranks, count * es, false);
    case COLL_ALGO_RING: return ring_form(nranks, count * es, vec);
    case COLL_ALGO_RING_LL: return vec ? COLL_ALGO_RING_LL : COLL_ALGO_RING_STEPS;
    case COLL_ALGO_TWOSHOT_LL: return vec ? COLL_ALGO_TWOSHOT_LL : COLL_ALGO_TWOSHOT;
    case COLL_ALGO_TWOSHOT_LL128: return vec ? COLL_ALGO_TWOSHOT_LL128 : COLL_ALGO_TWOSHOT;
    case COLL_ALGO_RING_CLUSTER:
      return vec && ring_cluster_supported(nranks) ? COLL_ALGO_RING_CLUSTER : COLL_ALGO_RING_STEPS;
    case COLL_ALGO_RING_CTA: return vec && ring_cta_supported(nranks) ? COLL_ALGO_RING_CTA : COLL_ALGO_RING_STEPS;
    case COLL_ALGO_RING_LANE: return vec && ring_lane_supported(nranks) ? COLL_ALGO_RING_LANE : COLL_ALGO_RING_STEPS;
    case COLL_ALGO_RING_WIRE: return vec && ring_cta_supported(nranks) ? COLL_ALGO_RING_WIRE : COLL_ERR_UNSUPPORTED;
    default: return algo;
  }
}

int coll_all_reduce(const void* const* send, void* const* recv, int nranks, size_t count, coll_dtype_t dtype,
                    coll_op_t op, coll_algo_t algo, void* workspace, size_t workspace_bytes, coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!valid_op(op) || algo < COLL_ALGO_AUTO || algo > COLL_ALGO_RING_WIRE) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || !all_nonnull(send, nranks) || !all_nonnull(recv, nranks)) return COLL_ERR_INVALID_ARG;
  const size_t bytes = count * es;
  if (bytes == 0) return COLL_OK;
  if (algo == COLL_ALGO_AUTO) {
    bool in_place = false;
    for (int r = 0; r < nranks; ++r) in_place = in_place || recv[r] == send[r];
    algo = auto_form(nranks, bytes, in_place);
  }
  if (!outputs_disjoint(recv, nranks, bytes)) return COLL_ERR_ALIAS;
  for (int q = 0; q < nranks; ++q)
    for (int r = 0; r < nranks; ++r)
      if (overlap(recv[q], bytes, send[r], bytes) && !(q == r && recv[q] == send[r] && algo != COLL_ALGO_ONESHOT))
        return COLL_ERR_ALIAS;
  const bool ws_needed = algo == COLL_ALGO_RING || algo == COLL_ALGO_RING_LL || algo == COLL_ALGO_RING_STEPS ||
                         algo == COLL_ALGO_TWOSHOT_LL || algo == COLL_ALGO_TWOSHOT_LL128;
  const bool packet_ws = algo == COLL_ALGO_RING_LL || algo == COLL_ALGO_TWOSHOT_LL ||
                         algo == COLL_ALGO_TWOSHOT_LL128;  // LL FIFOs: 256-byte aligned
  if (ws_needed && nranks > 1) {
    const size_t need = coll_all_reduce_workspace_size(nranks, count, dtype, algo);
    if (workspace == nullptr || workspace_bytes < need || (U(workspace) & (packet_ws ? 255 : 15)))
      return COLL_ERR_WORKSPACE;
    // the partials / FIFOs must not live inside any rank's buffer
    for (int r = 0; r < nranks; ++r)
      if (overlap(workspace, need, send[r], bytes) || overlap(workspace, need, recv[r], bytes)) return COLL_ERR_ALIAS;
  }
  if (nranks == 1) return copy_one(send[0], recv[0], bytes, S(stream));
  bool vec = true;
  for (int r = 0; r < nranks; ++r) vec = vec && al16(send[r]) && al16(recv[r]);
  const size_t seg = seg_elems(count, nranks, es);
  if (algo == COLL_ALGO_RING) algo = ring_form(nranks, bytes, vec);  // workspace checked above
  if (algo == COLL_ALGO_RING_WIRE) {  // one launch only: there is no stream-ordered form with rounded partials
    if (!vec || !ring_cta_supported(nranks)) return COLL_ERR_UNSUPPORTED;
    const char* in[COLL_MAX_RANKS];
    char* out[COLL_MAX_RANKS];
    for (int r = 0; r < nranks; ++r) {
      in[r] = static_cast<const char*>(send[r]);
      out[r] = static_cast<char*>(recv[r]);
    }
    return launch_ring_cta(in, out, nranks, count, dtype, op, true, S(stream));
  }
  if (algo == COLL_ALGO_RING_CLUSTER || algo == COLL_ALGO_RING_CTA || algo == COLL_ALGO_RING_LANE) {
    const bool has_ws = workspace != nullptr && workspace_bytes >= 24;
    const bool cta = algo == COLL_ALGO_RING_CTA;
    const bool lane = algo == COLL_ALGO_RING_LANE;
    if (vec && (lane  ? ring_lane_supported(nranks)
                : cta ? ring_cta_supported(nranks)
                      : ring_cluster_supported(nranks))) {
      if (has_ws && !al16(workspace)) return COLL_ERR_WORKSPACE;
      for (int r = 0; r < nranks && has_ws; ++r)
        if (overlap(workspace, 24, send[r], bytes) || overlap(workspace, 24, recv[r], bytes)) return COLL_ERR_ALIAS;
      const char* in[COLL_MAX_RANKS];
      char* out[COLL_MAX_RANKS];
      for (int r = 0; r < nranks; ++r) {
        in[r] = static_cast<const char*>(send[r]);
        out[r] = static_cast<char*>(recv[r]);
      }
      int* status = has_ws ? reinterpret_cast<int*>(static_cast<char*>(workspace) + 16) : nullptr;
      if (lane) return launch_ring_lane(in, out, nranks, count, dtype, op, S(stream));
      return cta ? launch_ring_cta(in, out, nranks, count, dtype, op, false, S(stream))
                 : launch_ring_cluster(in, out, nranks, count, dtype, op, status, S(stream));
    }
    // no one-launch form: the stream-ordered steps, given a RING-sized workspace
    const size_t need = 256 + ring_ws(count);
    if (workspace == nullptr || workspace_bytes < need || !al16(workspace)) return COLL_ERR_UNSUPPORTED;
    for (int r = 0; r < nranks; ++r)
      if (overlap(workspace, need, send[r], bytes) || overlap(workspace, need, recv[r], bytes)) return COLL_ERR_ALIAS;
    algo = COLL_ALGO_RING_STEPS;
  }
  if (algo == COLL_ALGO_RING_LL) {
    if (vec) {
      const char* in[COLL_MAX_RANKS];
      char* out[COLL_MAX_RANKS];
      for (int r = 0; r < nranks; ++r) {
        in[r] = static_cast<const char*>(send[r]);
        out[r] = static_cast<char*>(recv[r]);
      }
      int* status = reinterpret_cast<int*>(static_cast<char*>(workspace) + 16);
      return launch_ring_ll(in, out, nranks, count, dtype, op, workspace, status, S(stream));
    }
    algo = COLL_ALGO_RING_STEPS;  // unaligned buffers: the stream-ordered steps, partials after the header
  }
  if (algo == COLL_ALGO_TWOSHOT_LL128) {
    if (vec) {
      const char* in[COLL_MAX_RANKS];
      char* out[COLL_MAX_RANKS];
      for (int r = 0; r < nranks; ++r) {
        in[r] = static_cast<const char*>(send[r]);
        out[r] = static_cast<char*>(recv[r]);
      }
      int* status = reinterpret_cast<int*>(static_cast<char*>(workspace) + 16);
      return launch_twoshot_ll128(in, out, nranks, count, dtype, op, workspace, status, S(stream));
    }
    algo = COLL_ALGO_TWOSHOT;  // unaligned buffers: the plain two-shot kernel, the same result
  }
  if (algo == COLL_ALGO_TWOSHOT_LL) {
    if (vec) {
      const char* in[COLL_MAX_RANKS];
      char* out[COLL_MAX_RANKS];
      for (int r = 0; r < nranks; ++r) {
        in[r] = static_cast<const char*>(send[r]);
        out[r] = static_cast<char*>(recv[r]);
      }
      int* status = reinterpret_cast<int*>(static_cast<char*>(workspace) + 16);
      return launch_twoshot_ll(in, out, nranks, count, dtype, op, workspace, status, S(stream));
    }
    algo = COLL_ALGO_TWOSHOT;  // unaligned buffers: the plain two-shot kernel, the same result
  }
  if (algo == COLL_ALGO_RING_STEPS) {
    const char* in[COLL_MAX_RANKS];
    char* out[COLL_MAX_RANKS];
    for (int r = 0; r < nranks; ++r) {
      in[r] = static_cast<const char*>(send[r]);
      out[r] = static_cast<char*>(recv[r]);
    }
    // partials after the 256-byte header
    return launch_ring_steps(in, out, nranks, count, dtype, op, static_cast<char*>(workspace) + 256, vec, S(stream));
  }
  ReduceArgs a{};
  for (int r = 0; r < nranks; ++r) {
    a.in[r] = static_cast<const char*>(send[r]);
    a.out[r] = static_cast<char*>(recv[r]);
  }
  a.count = count;
  a.nin = nranks;
  a.nout = nranks;
  a.nslices = nranks;
  if (algo == COLL_ALGO_ONESHOT) {
    a.seg = count;
    const int bps = blocks_per_slice(vec ? bytes / 16 : count, nranks);
    return launch_reduce(a, dtype, op, kOneShot, vec, bps, S(stream));
  }
  a.seg = seg;
  const int bps = blocks_per_slice(vec ? seg * es / 16 : seg, nranks);
  return launch_reduce(a, dtype, op, kAll, vec, bps, S(stream));
}

// ------------------------------------------------------------- AllGather ----
int coll_all_gather(const void* const* send, void* const* recv, int nranks, size_t send_count, coll_dtype_t dtype,
                    coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || !all_nonnull(send, nranks) || !all_nonnull(recv, nranks)) return COLL_ERR_INVALID_ARG;
  const size_t blk = send_count * es;
  if (blk == 0) return COLL_OK;
  const size_t total = blk * nranks;
  if (!outputs_disjoint(recv, nranks, total)) return COLL_ERR_ALIAS;
  bool all_in_place = true;
  for (int r = 0; r < nranks; ++r) {
    const bool in_place = send[r] == static_cast<char*>(recv[r]) + static_cast<size_t>(r) * blk;
    all_in_place = all_in_place && in_place;
    for (int q = 0; q < nranks; ++q)
      if (overlap(send[r], blk, recv[q], total) && !(q == r && in_place)) return COLL_ERR_ALIAS;
  }
  FanoutArgs a{};
  for (int r = 0; r < nranks; ++r) {
    a.src[r] = static_cast<const char*>(send[r]);
    a.dst[r] = static_cast<char*>(recv[r]);
  }
  a.ns = nranks;
  a.nd = nranks;
  a.bytes = blk;
  a.dst_stride = blk;
  a.skip_diag = all_in_place ? 1 : 0;  // a partly in-place call copies those blocks onto themselves
  return launch_fanout(a, S(stream));
}

// ------------------------------------------------------------ All-to-All ----
int coll_all_to_all(const void* const* send, void* const* recv, int nranks, size_t count, coll_dtype_t dtype,
                    coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || !all_nonnull(send, nranks) || !all_nonnull(recv, nranks)) return COLL_ERR_INVALID_ARG;
  const size_t blk = count * es;
  if (blk == 0) return COLL_OK;
  const size_t total = blk * nranks;
  if (!outputs_disjoint(recv, nranks, total)) return COLL_ERR_ALIAS;
  for (int d = 0; d < nranks; ++d)
    for (int s = 0; s < nranks; ++s)
      if (overlap(recv[d], total, send[s], total)) return COLL_ERR_ALIAS;
  std::vector<CopyJob> jobs;
  jobs.reserve(static_cast<size_t>(nranks) * nranks);
  for (int s = 0; s < nranks; ++s)
    for (int d = 0; d < nranks; ++d)
      jobs.push_back({static_cast<const char*>(send[s]) + static_cast<size_t>(d) * blk,
                      static_cast<char*>(recv[d]) + static_cast<size_t>(s) * blk, blk});
  return launch_copy_jobs(jobs.data(), static_cast<int>(jobs.size()), S(stream));
}

int coll_all_to_all_v(const void* const* send, void* const* recv, int nranks, const int64_t* send_counts,
                      const int64_t* send_displs, const int64_t* recv_displs, const int64_t* send_capacity,
                      const int64_t* recv_capacity, size_t row_elems, coll_dtype_t dtype, coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || !all_nonnull(send, nranks) || !all_nonnull(recv, nranks) || !send_counts ||
      !send_displs || !recv_displs)
    return COLL_ERR_INVALID_ARG;
  const size_t row = row_elems * es;
  if (row == 0) return COLL_OK;
  const int n = nranks;
  std::vector<int64_t> recv_end(n, 0), send_end(n, 0);
  for (int s = 0; s < n; ++s)
    for (int d = 0; d < n; ++d) {
      const int64_t c = send_counts[s * n + d], so = send_displs[s * n + d], ro = recv_displs[d * n + s];
      if (c < 0 || so < 0 || ro < 0) return COLL_ERR_INVALID_ARG;
      if (c == 0) continue;
      send_end[s] = std::max(send_end[s], so + c);
      recv_end[d] = std::max(recv_end[d], ro + c);
      if (send_capacity && so + c > send_capacity[s]) return COLL_ERR_INVALID_ARG;
      if (recv_capacity && ro + c > recv_capacity[d]) return COLL_ERR_INVALID_ARG;
    }
  // receive blocks of one destination must not overlap each other
  for (int d = 0; d < n; ++d) {
    std::vector<std::pair<int64_t, int64_t>> iv;
    for (int s = 0; s < n; ++s)
      if (send_counts[s * n + d] > 0) iv.push_back({recv_displs[d * n + s], recv_displs[d * n + s] + send_counts[s * n + d]});
    std::sort(iv.begin(), iv.end());
    for (size_t i = 1; i < iv.size(); ++i)
      if (iv[i].first < iv[i - 1].second) return COLL_ERR_ALIAS;
  }
  for (int d = 0; d < n; ++d)
    for (int e = 0; e < n; ++e) {
      if (e > d && overlap(recv[d], recv_end[d] * row, recv[e], recv_end[e] * row)) return COLL_ERR_ALIAS;
      if (overlap(recv[d], recv_end[d] * row, send[e], send_end[e] * row)) return COLL_ERR_ALIAS;
    }
  std::vector<CopyJob> jobs;
  jobs.reserve(static_cast<size_t>(n) * n);
  for (int s = 0; s < n; ++s)
    for (int d = 0; d < n; ++d) {
      const int64_t c = send_counts[s * n + d];
      if (c == 0) continue;
      jobs.push_back({static_cast<const char*>(send[s]) + static_cast<size_t>(send_displs[s * n + d]) * row,
                      static_cast<char*>(recv[d]) + static_cast<size_t>(recv_displs[d * n + s]) * row,
                      static_cast<size_t>(c) * row});
    }
  return launch_copy_jobs(jobs.data(), static_cast<int>(jobs.size()), S(stream));
}

int coll_wait_flag(const uint32_t* flag, uint32_t expect, uint32_t budget_us, int* d_status, coll_stream_t stream) {
  if (flag == nullptr || d_status == nullptr || budget_us == 0 || budget_us > 10000000u) return COLL_ERR_INVALID_ARG;
  return launch_wait_flag(flag, expect, budget_us, d_status, S(stream));
}

// --------------------------------------------------------------- packets ----
size_t coll_packed_bytes(size_t bytes, coll_proto_t proto) {
  switch (proto) {
    case COLL_PROTO_SIMPLE: return bytes;
    case COLL_PROTO_LL: return 8 * ((bytes + 3) / 4);
    case COLL_PROTO_LL128: return 128 * ((bytes + 119) / 120);
  }
  return 0;
}

static bool valid_step(coll_proto_t proto, uint64_t step) {
  if (step == 0) return false;
  if (proto == COLL_PROTO_LL && static_cast<uint32_t>(step) == 0) return false;
  return true;
}

int coll_ll_pack(const void* src, void* packed, size_t bytes, coll_proto_t proto, uint64_t step, coll_stream_t stream) {
  return coll_ll_pack_ranks(&src, &packed, 1, bytes, proto, step, stream);
}

int coll_ll_unpack(const void* packed, void* dst, size_t bytes, coll_proto_t proto, uint64_t step, int* d_status,
                   coll_stream_t stream) {
  return coll_ll_unpack_ranks(&packed, &dst, 1, bytes, proto, step, d_status, stream);
}

// the n messages (`mbytes` each) and the n packet buffers (`pbytes` each):
// no message overlaps any packet buffer, and the written side's buffers are
// disjoint
static int codec_check(const void* const* msgs, const void* const* pkts, int n, size_t mbytes, size_t pbytes,
                       bool pack) {
  for (int r = 0; r < n; ++r)
    if (!al16(pkts[r])) return COLL_ERR_INVALID_ARG;
  for (int r = 0; r < n; ++r)
    for (int q = 0; q < n; ++q) {
      if (overlap(msgs[r], mbytes, pkts[q], pbytes)) return COLL_ERR_ALIAS;
      if (q != r && (pack ? overlap(pkts[r], pbytes, pkts[q], pbytes) : overlap(msgs[r], mbytes, msgs[q], mbytes)))
        return COLL_ERR_ALIAS;
    }
  return COLL_OK;
}

int coll_ll_pack_ranks(const void* const* src, void* const* packed, int nranks, size_t bytes, coll_proto_t proto,
                       uint64_t step, coll_stream_t stream) {
  if (proto != COLL_PROTO_LL && proto != COLL_PROTO_LL128) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || !all_nonnull(src, nranks) || !all_nonnull(packed, nranks) || !valid_step(proto, step))
    return COLL_ERR_INVALID_ARG;
  const int c = codec_check(src, packed, nranks, bytes, coll_packed_bytes(bytes, proto), true);
  if (c != COLL_OK) return c;
  if (bytes == 0) return COLL_OK;
  CodecArgs a{};
  for (int r = 0; r < nranks; ++r) {
    a.in[r] = static_cast<const uint8_t*>(src[r]);
    a.out[r] = static_cast<uint8_t*>(packed[r]);
  }
  a.bytes = bytes;
  a.step = step;
  a.n = nranks;
  return launch_ll_pack(a, proto, S(stream));
}

int coll_ll_unpack_ranks(const void* const* packed, void* const* dst, int nranks, size_t bytes, coll_proto_t proto,
                         uint64_t step, int* d_status, coll_stream_t stream) {
  if (proto != COLL_PROTO_LL && proto != COLL_PROTO_LL128) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || !all_nonnull(packed, nranks) || !all_nonnull(dst, nranks) || !valid_step(proto, step))
    return COLL_ERR_INVALID_ARG;
  const int c = codec_check(dst, packed, nranks, bytes, coll_packed_bytes(bytes, proto), false);
  if (c != COLL_OK) return c;
  if (bytes == 0) return COLL_OK;
  CodecArgs a{};
  for (int r = 0; r < nranks; ++r) {
    a.in[r] = static_cast<const uint8_t*>(packed[r]);
    a.out[r] = static_cast<uint8_t*>(dst[r]);
  }
  a.bytes = bytes;
  a.step = step;
  a.n = nranks;
  a.status = d_status;
  return launch_ll_unpack(a, proto, S(stream));
}

int coll_all_reduce_packed(const void* const* packed_in, void* const* packed_out, int nranks, size_t count,
                           coll_dtype_t dtype, coll_op_t op, coll_proto_t proto, uint64_t step, int* d_status,
                           coll_stream_t stream) {
  if (proto == COLL_PROTO_SIMPLE)
    return coll_all_reduce(packed_in, packed_out, nranks, count, dtype, op, COLL_ALGO_TWOSHOT, nullptr, 0, stream);
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!valid_op(op) || (proto != COLL_PROTO_LL && proto != COLL_PROTO_LL128)) return COLL_ERR_UNSUPPORTED;
  if (!valid_n(nranks) || !all_nonnull(packed_in, nranks) || !all_nonnull(packed_out, nranks) ||
      !valid_step(proto, step))
    return COLL_ERR_INVALID_ARG;
  const size_t payload = count * es;
  if (payload == 0) return COLL_OK;
  const size_t pbytes = coll_packed_bytes(payload, proto);
  for (int r = 0; r < nranks; ++r)
    if (!al16(packed_in[r]) || !al16(packed_out[r])) return COLL_ERR_INVALID_ARG;
  if (!outputs_disjoint(packed_out, nranks, pbytes)) return COLL_ERR_ALIAS;
  for (int q = 0; q < nranks; ++q)
    for (int r = 0; r < nranks; ++r)
      if (overlap(packed_out[q], pbytes, packed_in[r], pbytes) && !(q == r && packed_out[q] == packed_in[r]))
        return COLL_ERR_ALIAS;
  PackedReduceArgs a{};
  for (int r = 0; r < nranks; ++r) {
    a.in[r] = static_cast<const char*>(packed_in[r]);
    a.out[r] = static_cast<char*>(packed_out[r]);
  }
  a.nlines = pbytes / (proto == COLL_PROTO_LL ? 8 : 128);
  a.payload_bytes = payload;
  a.step = step;
  a.n = nranks;
  a.status = d_status;
  return launch_all_reduce_packed(a, dtype, op, proto, S(stream));
}

// ------------------------------------------------------------------- MoE ----
static bool moe_shape_ok(int nranks, int tokens, int topk, int n_experts) {
  if (!valid_n(nranks) || tokens < 0 || topk < 1 || topk > 32) return false;
  if (n_experts < nranks || n_experts > COLL_MAX_EXPERTS || n_experts % nranks != 0) return false;
  if (static_cast<int64_t>(nranks) * tokens * topk >= (int64_t{1} << 31)) return false;
  return true;
}

size_t coll_moe_route_workspace_size(int nranks, int tokens, int topk, int n_experts) {
  if (!moe_shape_ok(nranks, tokens, topk, n_experts)) return 0;
  return moe_route_workspace(nranks, tokens, topk, n_experts);
}

static int moe_route_impl(const int32_t* const* topk_ids, int nranks, int tokens, int topk, int n_experts,
                          int64_t* d_send_counts, int64_t* d_send_displs, int64_t* d_recv_displs,
                          int32_t* const* d_pos, int* d_status, void* workspace, size_t workspace_bytes,
                          coll_stream_t stream, bool dedup) {
  if (!moe_shape_ok(nranks, tokens, topk, n_experts)) return COLL_ERR_INVALID_ARG;
  if (topk_ids == nullptr || d_pos == nullptr || !d_send_counts || !d_send_displs || !d_recv_displs)
    return COLL_ERR_INVALID_ARG;
  // with no tokens the per-rank arrays are empty and never touched
  if (tokens > 0 && (!all_nonnull(topk_ids, nranks) || !all_nonnull(d_pos, nranks))) return COLL_ERR_INVALID_ARG;
  const size_t need = moe_route_workspace(nranks, tokens, topk, n_experts);
  if (workspace == nullptr || workspace_bytes < need || (U(workspace) & 255) != 0) return COLL_ERR_WORKSPACE;
  MoeRouteArgs a{};
  for (int r = 0; r < nranks; ++r) {
    a.ids[r] = topk_ids[r];
    a.pos[r] = d_pos[r];
  }
  a.send_counts = d_send_counts;
  a.send_displs = d_send_displs;
  a.recv_displs = d_recv_displs;
  a.n = nranks;
  a.tokens = tokens;
  a.topk = topk;
  a.n_experts = n_experts;
  a.tiles = std::max(1, (tokens + 255) / 256);
  a.dedup = dedup ? 1 : 0;
  a.buckets = dedup ? nranks : n_experts;
  a.bpr = dedup ? 1 : n_experts / nranks;
  // the layout of the per-expert route; the deduplicated one uses a prefix of each array
  const size_t cells = static_cast<size_t>(nranks) * n_experts * a.tiles;
  a.tile_cnt = static_cast<int32_t*>(workspace);
  a.tile_base = reinterpret_cast<int64_t*>(static_cast<char*>(workspace) + (cells * 4 + 255) / 256 * 256);
  a.status = d_status;
  return launch_moe_route(a, S(stream));
}

int coll_moe_route(const int32_t* const* topk_ids, int nranks, int tokens, int topk, int n_experts,
                   int64_t* d_send_counts, int64_t* d_send_displs, int64_t* d_recv_displs, int32_t* const* d_pos,
                   int* d_status, void* workspace, size_t workspace_bytes, coll_stream_t stream) {
  return moe_route_impl(topk_ids, nranks, tokens, topk, n_experts, d_send_counts, d_send_displs, d_recv_displs, d_pos,
                        d_status, workspace, workspace_bytes, stream, false);
}

int coll_moe_route_dedup(const int32_t* const* topk_ids, int nranks, int tokens, int topk, int n_experts,
                         int64_t* d_send_counts, int64_t* d_send_displs, int64_t* d_recv_displs,
                         int32_t* const* d_pos, int* d_status, void* workspace, size_t workspace_bytes,
                         coll_stream_t stream) {
  return moe_route_impl(topk_ids, nranks, tokens, topk, n_experts, d_send_counts, d_send_displs, d_recv_displs, d_pos,
                        d_status, workspace, workspace_bytes, stream, true);
}

int coll_moe_dispatch(const void* const* x, const int32_t* const* topk_ids, const int32_t* const* d_pos,
                      void* const* recv, int nranks, int tokens, int topk, int n_experts, size_t hidden,
                      coll_dtype_t dtype, int64_t recv_capacity_rows, int* d_status, coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es) return COLL_ERR_UNSUPPORTED;
  if (!moe_shape_ok(nranks, tokens, topk, n_experts) || recv_capacity_rows < 0) return COLL_ERR_INVALID_ARG;
  if (!all_nonnull(x, nranks) || !all_nonnull(topk_ids, nranks) || !all_nonnull(d_pos, nranks) ||
      !all_nonnull(recv, nranks))
    return COLL_ERR_INVALID_ARG;
  const size_t row = hidden * es;
  if (row == 0 || tokens == 0) return COLL_OK;
  const size_t in_bytes = row * tokens, out_bytes = row * static_cast<size_t>(recv_capacity_rows);
  if (!outputs_disjoint(recv, nranks, out_bytes)) return COLL_ERR_ALIAS;
  for (int d = 0; d < nranks; ++d)
    for (int s = 0; s < nranks; ++s)
      if (overlap(recv[d], out_bytes, x[s], in_bytes)) return COLL_ERR_ALIAS;
  MoeMoveArgs a{};
  for (int r = 0; r < nranks; ++r) {
    a.x[r] = static_cast<const char*>(x[r]);
    a.y[r] = static_cast<char*>(recv[r]);
    a.ids[r] = topk_ids[r];
    a.pos[r] = d_pos[r];
  }
  a.row_bytes = row;
  a.capacity = recv_capacity_rows;
  a.status = d_status;
  a.n = nranks;
  a.tokens = tokens;
  a.topk = topk;
  a.epr = n_experts / nranks;
  return launch_moe_dispatch(a, S(stream));
}

int coll_moe_combine(const void* const* y, const int32_t* const* topk_ids, const int32_t* const* d_pos,
                     const float* const* topk_w, void* const* out, int nranks, int tokens, int topk, int n_experts,
                     size_t hidden, coll_dtype_t dtype, int64_t recv_capacity_rows, int* d_status,
                     coll_stream_t stream) {
  const int es = elem_size(dtype);
  if (!es || dtype == COLL_INT32) return COLL_ERR_UNSUPPORTED;
  if (!moe_shape_ok(nranks, tokens, topk, n_experts) || recv_capacity_rows < 0) return COLL_ERR_INVALID_ARG;
  if (!all_nonnull(y, nranks) || !all_nonnull(topk_ids, nranks) || !all_nonnull(d_pos, nranks) ||
      !all_nonnull(topk_w, nranks) || !all_nonnull(out, nranks))
    return COLL_ERR_INVALID_ARG;
  const size_t row = hidden * es;
  if (row == 0 || tokens == 0) return COLL_OK;
  const size_t out_bytes = row * tokens, in_bytes = row * static_cast<size_t>(recv_capacity_rows);
  if (!outputs_disjoint(out, nranks, out_bytes)) return COLL_ERR_ALIAS;
  for (int d = 0; d < nranks; ++d)
    for (int s = 0; s < nranks; ++s)
      if (overlap(out[d], out_bytes, y[s], in_bytes)) return COLL_ERR_ALIAS;
  MoeMoveArgs a{};
  for (int r = 0; r < nranks; ++r) {
    a.x[r] = static_cast<const char*>(y[r]);
    a.y[r] = static_cast<char*>(out[r]);
    a.ids[r] = topk_ids[r];
    a.pos[r] = d_pos[r];
    a.w[r] = topk_w[r];
  }
  a.row_bytes = row;
  a.capacity = recv_capacity_rows;
  a.status = d_status;
  a.n = nranks;
  a.tokens = tokens;
  a.topk = topk;
  a.epr = n_experts / nranks;
  return launch_moe_combine(a, dtype, S(stream));
}

}  // extern "C"
