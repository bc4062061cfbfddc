// Movement kernels: bit copies between virtual-rank buffers.
//
//  k_fanout      one read, many writes: broadcast (vLLM collectives tutorial
//                section 1.1) and all-gather (section 7.1) read every source
//                element once and store it to every destination.
//  k_copy_jobs   a list of independent 1-D copies, partitioned over the grid
//                by byte ranges so that very unequal blocks (all-to-all-v,
//                section 8.2) still spread evenly: scatter, flat gather,
//                all-to-all, all-to-all-v and the ring's all-gather steps.
//  k_gather_rows the last-dimension gather of section 2.2.1: rank r's
//                [rows, cols] block lands at columns [r*cols, (r+1)*cols).
//
// All three move 16-byte units when every address and length allows it and
// fall back to narrower units otherwise.
#include <algorithm>
#include <vector>

#include "bulk.cuh"
#include "common.cuh"
#include "internal.h"

namespace mvr {

// The fan-out and the copy lists use bulk copies from this many tiles per
// resident CTA (6 per SM) up; below that the element path is faster.
constexpr uint64_t kTmaMinTilesPerCta = 4;

static int pick_unit(uint64_t bits) {
  // largest power of two <= 16 that divides every address / length OR-ed into `bits`
  if ((bits & 15) == 0) return 16;
  if ((bits & 7) == 0) return 8;
  if ((bits & 3) == 0) return 4;
  if ((bits & 1) == 0) return 2;
  return 1;
}

// one unit per thread for each of `slices` slices, the slices interleaved
static unsigned grid_for(uint64_t units, int slices) {
  const uint64_t per = std::min<uint64_t>(stream_grid(units, kThreads), kMaxStreamGrid / std::max(1, slices));
  return static_cast<unsigned>(per * slices);
}

// ------------------------------------------------------------- fan-out ----

template <int U>
__global__ void __launch_bounds__(kThreads) k_fanout(const __grid_constant__ FanoutArgs a) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x % a.ns;
  const int part = blockIdx.x / a.ns;
  const int parts = gridDim.x / a.ns;
  const uint64_t units = a.bytes / U;
  const uint64_t stride = static_cast<uint64_t>(parts) * blockDim.x;
  const char* src = a.src[r];
  const uint64_t roff = static_cast<uint64_t>(r) * a.dst_stride;
  for (uint64_t u = static_cast<uint64_t>(part) * blockDim.x + threadIdx.x; u < units; u += stride) {
    const auto x = ldu<U>(src + u * U);
#pragma unroll 8
    for (int q = 0; q < a.nd; ++q) {
      if (a.skip_diag && q == r) continue;
      stu<U>(a.dst[q] + roff + u * U, x);
    }
  }
  if (part == 0) {  // bytes beyond the last whole unit
    const uint64_t b = units * U + threadIdx.x;
    if (b < a.bytes) {
      const char x = src[b];
      for (int q = 0; q < a.nd; ++q) {
        if (a.skip_diag && q == r) continue;
        a.dst[q][roff + b] = x;
      }
    }
  }
}

// Bulk-copy fan-out: one thread per CTA streams tiles of a source into a ring
// of shared-memory stages with cp.async.bulk and writes each landed tile to
// every destination with bulk stores; a stage is refilled once its stores
// have finished reading it.  Tiles of all sources are interleaved over the
// grid so that every source progresses at once.  The grid has one CTA per
// kTmaTilesPerCta tiles (CTA b takes tiles b and b + G), launched in order,
// so a CTA's loads are all in flight at once and the next CTAs' loads
// overlap its stores: measured faster than a resident grid walking every
// tile (all 8 sources of 16 MiB to 8 ranks: 191 against 217 us; 4 tiles per
// CTA 193).
constexpr int kTmaTile = 8192;
// A CTA fills kTmaTilesPerCta of its 4 stages; all 4 serve when the grid is
// capped and CTAs walk more tiles.  Sizing the shared memory for 2 stages
// instead (more CTAs resident per SM) measured slower: 192.5 against 190.5 us.
constexpr int kTmaStages = 4;
constexpr uint64_t kTmaTilesPerCta = 2;

__global__ void __launch_bounds__(32) k_fanout_tma(const __grid_constant__ FanoutArgs a) {
  extern __shared__ __align__(128) unsigned char stage_buf[];
  __shared__ __align__(8) uint64_t bar[kTmaStages];
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x != 0) return;
  for (int st = 0; st < kTmaStages; ++st) mbar_init(&bar[st], 1);
  fence_barrier_init();
  const uint64_t pieces = (a.bytes + kTmaTile - 1) / kTmaTile;
  const uint64_t total = pieces * static_cast<uint64_t>(a.ns);
  const uint64_t stride = gridDim.x;
  auto issue = [&](uint64_t t, int st) {
    const int r = static_cast<int>(t % a.ns);
    const uint64_t off = (t / a.ns) * kTmaTile;
    const uint32_t len = static_cast<uint32_t>(a.bytes - off < kTmaTile ? a.bytes - off : kTmaTile);
    mbar_arrive_expect_tx(&bar[st], len);
    bulk_load(stage_buf + st * kTmaTile, a.src[r] + off, len, &bar[st]);
  };
  int inflight = 0;
  for (int st = 0; st < kTmaStages && blockIdx.x + st * stride < total; ++st, ++inflight) issue(blockIdx.x + st * stride, st);
  int i = 0;
  for (uint64_t t = blockIdx.x; t < total; t += stride, ++i) {
    const int st = i % kTmaStages;
    if (!mbar_wait_bounded(&bar[st], (i / kTmaStages) & 1)) {
      report(a.status, COLL_DEV_TIMEOUT, 1);
      bulk_wait_all();
      for (int k = 1; k < inflight; ++k)  // the loads still in flight, bounded again
        mbar_wait_bounded(&bar[(i + k) % kTmaStages], ((i + k) / kTmaStages) & 1);
      return;
    }
    --inflight;
    const int r = static_cast<int>(t % a.ns);
    const uint64_t off = (t / a.ns) * kTmaTile;
    const uint32_t len = static_cast<uint32_t>(a.bytes - off < kTmaTile ? a.bytes - off : kTmaTile);
    const unsigned char* src = stage_buf + st * kTmaTile;
    const uint64_t roff = static_cast<uint64_t>(r) * a.dst_stride + off;
    for (int q = 0; q < a.nd; ++q) {
      if (a.skip_diag && q == r) continue;
      bulk_store(a.dst[q] + roff, src, len);
    }
    bulk_commit();
    const uint64_t nxt = t + kTmaStages * stride;
    if (nxt < total) {
      bulk_wait_read<0>();
      issue(nxt, st);
      ++inflight;
    }
  }
  bulk_wait_all();
}

int launch_fanout(const FanoutArgs& a, cudaStream_t s) {
  if (a.bytes == 0 || a.ns == 0 || a.nd == 0) return COLL_OK;
  uint64_t bits = a.dst_stride;
  for (int r = 0; r < a.ns; ++r) bits |= reinterpret_cast<uintptr_t>(a.src[r]);
  for (int q = 0; q < a.nd; ++q) bits |= reinterpret_cast<uintptr_t>(a.dst[q]);
  const uint64_t tiles = (a.bytes + kTmaTile - 1) / kTmaTile * a.ns;
  const uint64_t resident = static_cast<uint64_t>(num_sms()) * 6;  // 6 x 32 KB of stages per SM
  if ((bits & 15) == 0 && (a.bytes & 15) == 0 && tiles >= kTmaMinTilesPerCta * resident) {
    const uint64_t grid = stream_grid(tiles, kTmaTilesPerCta);
    launch_pdl(k_fanout_tma, dim3(static_cast<unsigned>(grid)), dim3(32), kTmaStages * kTmaTile, s, a);
    return launch_status(cudaGetLastError());
  }
  const int U = pick_unit(bits);
  const unsigned grid = grid_for(a.bytes / U, a.ns);
  switch (U) {
    case 16: launch_pdl(k_fanout<16>, dim3(grid), dim3(kThreads), 0, s, a); break;
    case 8: launch_pdl(k_fanout<8>, dim3(grid), dim3(kThreads), 0, s, a); break;
    case 4: launch_pdl(k_fanout<4>, dim3(grid), dim3(kThreads), 0, s, a); break;
    case 2: launch_pdl(k_fanout<2>, dim3(grid), dim3(kThreads), 0, s, a); break;
    default: launch_pdl(k_fanout<1>, dim3(grid), dim3(kThreads), 0, s, a); break;
  }
  return launch_status(cudaGetLastError());
}

// ------------------------------------------------------------ copy jobs ----

struct JobU {
  const char* src;
  char* dst;
  uint64_t start;  // first unit of this job in the concatenation of all jobs
};
constexpr int kMaxJobs = 960;  // 960 * 24 B + header < 32 KB of kernel parameters
struct CopyJobsArgs {
  uint64_t total;  // units over all jobs
  int njobs;
  JobU job[kMaxJobs + 1];  // job[njobs].start == total (sentinel)
};

template <int U>
__global__ void __launch_bounds__(kThreads) k_copy_jobs(const __grid_constant__ CopyJobsArgs a) {
  pdl_wait();
  pdl_trigger();
  // block b owns the contiguous unit range [b*total/B, (b+1)*total/B)
  const uint64_t B = gridDim.x;
  const uint64_t lo = a.total * blockIdx.x / B;
  const uint64_t hi = a.total * (blockIdx.x + 1) / B;
  if (lo >= hi) return;
  // first job holding `lo` (binary search; uniform over the block)
  int j0 = 0, j1 = a.njobs - 1;
  while (j0 < j1) {
    const int m = (j0 + j1 + 1) >> 1;
    if (a.job[m].start <= lo) j0 = m;
    else j1 = m - 1;
  }
  int j = j0;
  // four units per thread per round: all four loads are issued before any store
  constexpr int kU = 4;
  for (uint64_t base = lo + threadIdx.x; base < hi; base += kU * blockDim.x) {
    typename UnitT<U>::T v[kU];
    char* d[kU];
#pragma unroll
    for (int i = 0; i < kU; ++i) {
      const uint64_t u = base + static_cast<uint64_t>(i) * blockDim.x;
      d[i] = nullptr;
      if (u < hi) {
        while (u >= a.job[j + 1].start) ++j;
        const uint64_t off = (u - a.job[j].start) * U;
        v[i] = ldu<U>(a.job[j].src + off);
        d[i] = a.job[j].dst + off;
      }
    }
#pragma unroll
    for (int i = 0; i < kU; ++i)
      if (d[i] != nullptr) stu<U>(d[i], v[i]);
  }
}

// Bulk-copy form of the job list for large copies: one thread per CTA
// streams tiles (each within one job) through a ring of shared-memory stages,
// loading with cp.async.bulk and storing each landed tile with a bulk store.
struct TmaJob {
  const char* src;
  char* dst;
  uint64_t bytes;
  uint64_t tile0;  // first tile of this job in the concatenation of all jobs
};
constexpr int kMaxTmaJobs = 900;  // 900 * 32 B + header < 32 KB of kernel parameters
struct TmaJobsArgs {
  uint64_t total_tiles;
  int njobs;
  int* status;
  TmaJob job[kMaxTmaJobs + 1];  // job[njobs].tile0 == total_tiles (sentinel)
};

__global__ void __launch_bounds__(32) k_copy_jobs_tma(const __grid_constant__ TmaJobsArgs a) {
  extern __shared__ __align__(128) unsigned char stage_buf[];
  __shared__ __align__(8) uint64_t bar[kTmaStages];
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x != 0) return;
  for (int st = 0; st < kTmaStages; ++st) mbar_init(&bar[st], 1);
  fence_barrier_init();
  const uint64_t stride = gridDim.x;
  int jl = 0;  // job of the next tile to load (a CTA visits its tiles in increasing order)
  int js = 0;  // job of the next tile to store
  auto locate = [&](uint64_t t, int& j, uint64_t& off, uint32_t& len) {
    // binary search from j up (a CTA's tiles increase, so job[j].tile0 <= t);
    // a linear walk cost the 64-job all-to-all 13% (47.1 against 41.2 us)
    int hi = a.njobs;  // job[hi].tile0 > t (job[njobs] is the sentinel)
    while (hi - j > 1) {
      const int mid = (j + hi) >> 1;
      if (a.job[mid].tile0 <= t)
        j = mid;
      else
        hi = mid;
    }
    off = (t - a.job[j].tile0) * kTmaTile;
    const uint64_t rest = a.job[j].bytes - off;
    len = static_cast<uint32_t>(rest < kTmaTile ? rest : kTmaTile);
  };
  auto issue = [&](uint64_t t, int st) {
    uint64_t off;
    uint32_t len;
    locate(t, jl, off, len);
    mbar_arrive_expect_tx(&bar[st], len);
    bulk_load(stage_buf + st * kTmaTile, a.job[jl].src + off, len, &bar[st]);
  };
  int inflight = 0;
  for (int st = 0; st < kTmaStages && blockIdx.x + st * stride < a.total_tiles; ++st, ++inflight)
    issue(blockIdx.x + st * stride, st);
  int i = 0;
  for (uint64_t t = blockIdx.x; t < a.total_tiles; t += stride, ++i) {
    const int st = i % kTmaStages;
    if (!mbar_wait_bounded(&bar[st], (i / kTmaStages) & 1)) {
      report(a.status, COLL_DEV_TIMEOUT, 1);
      bulk_wait_all();
      for (int k = 1; k < inflight; ++k) mbar_wait_bounded(&bar[(i + k) % kTmaStages], ((i + k) / kTmaStages) & 1);
      return;
    }
    --inflight;
    uint64_t off;
    uint32_t len;
    locate(t, js, off, len);
    bulk_store(a.job[js].dst + off, stage_buf + st * kTmaTile, len);
    bulk_commit();
    const uint64_t nxt = t + kTmaStages * stride;
    if (nxt < a.total_tiles) {
      bulk_wait_read<0>();
      issue(nxt, st);
      ++inflight;
    }
  }
  bulk_wait_all();
}

int launch_copy_jobs(const CopyJob* jobs, int njobs, cudaStream_t s) {
  // drop empty jobs; choose one unit for all jobs of a launch
  std::vector<CopyJob> v;
  v.reserve(njobs);
  uint64_t bits = 0;
  for (int i = 0; i < njobs; ++i) {
    if (jobs[i].bytes == 0) continue;
    v.push_back(jobs[i]);
    bits |= reinterpret_cast<uintptr_t>(jobs[i].src) | reinterpret_cast<uintptr_t>(jobs[i].dst) | jobs[i].bytes;
  }
  if (v.empty()) return COLL_OK;
  const int U = pick_unit(bits);
  // large, 16-byte aligned job lists go through the bulk-copy path
  if (U == 16) {
    uint64_t tiles = 0;
    for (const CopyJob& j : v) tiles += (j.bytes + kTmaTile - 1) / kTmaTile;
    const uint64_t resident = static_cast<uint64_t>(num_sms()) * 6;
    if (tiles >= kTmaMinTilesPerCta * resident) {
      static thread_local TmaJobsArgs targs;  // ~29 KB: keep it off the stack
      for (size_t first = 0; first < v.size(); first += kMaxTmaJobs) {
        const int nj = static_cast<int>(std::min<size_t>(kMaxTmaJobs, v.size() - first));
        uint64_t acc = 0;
        for (int i = 0; i < nj; ++i) {
          const CopyJob& j = v[first + i];
          targs.job[i] = TmaJob{j.src, j.dst, j.bytes, acc};
          acc += (j.bytes + kTmaTile - 1) / kTmaTile;
        }
        targs.job[nj] = TmaJob{nullptr, nullptr, 0, acc};
        targs.total_tiles = acc;
        targs.njobs = nj;
        targs.status = nullptr;
        const uint64_t grid = stream_grid(acc, kTmaTilesPerCta);  // in order, as the fan-out
        launch_pdl(k_copy_jobs_tma, dim3(static_cast<unsigned>(grid)), dim3(32), kTmaStages * kTmaTile, s, targs);
        const int st = launch_status(cudaGetLastError());
        if (st != COLL_OK) return st;
      }
      return COLL_OK;
    }
  }
  static thread_local CopyJobsArgs args;  // ~23 KB: keep it off the stack
  for (size_t first = 0; first < v.size(); first += kMaxJobs) {
    const int nj = static_cast<int>(std::min<size_t>(kMaxJobs, v.size() - first));
    uint64_t acc = 0;
    for (int i = 0; i < nj; ++i) {
      args.job[i].src = v[first + i].src;
      args.job[i].dst = v[first + i].dst;
      args.job[i].start = acc;
      acc += v[first + i].bytes / U;
    }
    args.job[nj].src = nullptr;
    args.job[nj].dst = nullptr;
    args.job[nj].start = acc;
    args.total = acc;
    args.njobs = nj;
    void (*fn)(CopyJobsArgs) = U == 16 ? k_copy_jobs<16>
                              : U == 8  ? k_copy_jobs<8>
                              : U == 4  ? k_copy_jobs<4>
                              : U == 2  ? k_copy_jobs<2>
                                        : k_copy_jobs<1>;
    // about one unit per thread, CTAs launched in order
    launch_pdl(fn, dim3(static_cast<unsigned>(stream_grid(acc, kThreads))), dim3(kThreads), 0, s, args);
    const int st = launch_status(cudaGetLastError());
    if (st != COLL_OK) return st;
  }
  return COLL_OK;
}

// ---------------------------------------------------------- row gather ----

template <int U>
__global__ void __launch_bounds__(kThreads) k_gather_rows(const __grid_constant__ GatherRowsArgs a) {
  pdl_wait();
  pdl_trigger();
  // blockIdx.x = part * n + r ; parts stride over rows, threads over columns
  const int r = blockIdx.x % a.n;
  const int part = blockIdx.x / a.n;
  const int parts = gridDim.x / a.n;
  const uint64_t ru = a.row_bytes / U;
  const char* src = a.src[r];
  char* dst = a.dst + static_cast<uint64_t>(r) * a.row_bytes;
  for (uint64_t row = part; row < a.rows; row += parts) {
    const char* sp = src + row * a.row_bytes;
    char* dp = dst + row * a.dst_pitch;
    // four units in flight per thread, then their stores (44.0 -> 43.0 us for
    // 8 ranks x 256 rows of 64 KB against one load-store pair at a time)
    constexpr int kB = 4;
    uint64_t u = threadIdx.x;
    for (; u + (kB - 1) * blockDim.x < ru; u += kB * blockDim.x) {
      typename UnitT<U>::T x[kB];
#pragma unroll
      for (int k = 0; k < kB; ++k) x[k] = ldu<U>(sp + (u + k * blockDim.x) * U);
#pragma unroll
      for (int k = 0; k < kB; ++k) stu<U>(dp + (u + k * blockDim.x) * U, x[k]);
    }
    for (; u < ru; u += blockDim.x) stu<U>(dp + u * U, ldu<U>(sp + u * U));
  }
}

int launch_gather_rows(const GatherRowsArgs& a, cudaStream_t s) {
  if (a.rows == 0 || a.row_bytes == 0) return COLL_OK;
  uint64_t bits = a.row_bytes | a.dst_pitch | reinterpret_cast<uintptr_t>(a.dst);
  for (int r = 0; r < a.n; ++r) bits |= reinterpret_cast<uintptr_t>(a.src[r]);
  const int U = pick_unit(bits);
  void (*fn)(GatherRowsArgs) = U == 16 ? k_gather_rows<16>
                              : U == 8  ? k_gather_rows<8>
                              : U == 4  ? k_gather_rows<4>
                              : U == 2  ? k_gather_rows<2>
                                        : k_gather_rows<1>;
  // one CTA per row of every rank, launched in order: measured faster than 8
  // CTAs per SM walking the rows (44.0 against 45.0 us for 8 ranks x 256
  // rows of 64 KB) and than a resident-only grid (48.0 us)
  const uint64_t parts = std::min<uint64_t>(a.rows, kMaxStreamGrid / a.n);
  launch_pdl(fn, dim3(static_cast<unsigned>(parts * a.n)), dim3(kThreads), 0, s, a);
  return launch_status(cudaGetLastError());
}

}  // namespace mvr
