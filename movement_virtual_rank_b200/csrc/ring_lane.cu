// Ring all-reduce with the virtual ranks as lanes of one warp: the hop from
// rank r to rank r+1 is a warp shuffle, so the ring's 2N-2 steps run in
// registers with no shared memory, no barrier and nothing to wait on.
//
// The schedule, chunk order, fp32 partials and the single rounding are those
// of coll_all_reduce(RING) (TP communication essay, the ring's 2(N-1) steps;
// NCCL's ring kernel named in "From NCCL Ring LL to PCIe IPC AllReduce"), so
// the result is bit-identical.  A warp holds 32 / W ring instances of W
// lanes each (W = N rounded up to a power of two; lanes r >= N of an
// instance idle): lane r of instance g plays rank r for the 16-byte vector at
// column col = item * (32 / W) + g of every chunk.  A warp item is those
// 32 / W adjacent columns, so each load or store instruction of the warp
// touches 32 / W x 16 contiguous bytes of every rank's buffer.
//
// Steps of one instance (rank r, its predecessor r-1 mod N):
//   load     the vector of column col of every chunk, in the order the
//            reduce-scatter needs them: step k uses chunk (r - 1 - k) mod N;
//   RS       step 0 starts the partial from the chunk-(r-1) input; step k
//            (1..N-1) takes the predecessor's partial (fp32 / int32, VN
//            shuffles) and adds this rank's chunk-(r-1-k) input, so the
//            partial of chunk c visits ranks c+1, c+2, ..., c in ring order
//            and after N-1 steps rank r holds chunk r, rounded once;
//   AG       N-1 steps pass the rounded vector on (4 shuffles of 32 bits);
//            at step j rank r receives chunk (r - j) mod N and stores it.
// The next item's inputs are loaded as soon as this item's reduce-scatter
// has used its own, so they are in flight while the all-gather stores.
//
// Columns are whole 16-byte vectors of a chunk, and chunks are whole numbers
// of vectors, so every vector lies wholly inside the message or wholly
// outside it -- except the one holding the message's last count mod VN
// elements, which ring_tail() reduces at the end in that chunk's ring order.
// A vector's inside-ness is the same on every rank, so a partial either
// stays inside the message on its whole path or is never stored.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "ring_tail.cuh"

namespace mvr {

constexpr int kRlThreads = 128;
constexpr int kRlWarps = kRlThreads / 32;

struct RingLaneArgs {
  const char* in[kMaxRanks];
  char* out[kMaxRanks];
  uint64_t count, seg;  // elements of a rank's buffer, of a chunk (whole vectors)
  uint64_t cols;        // vectors per chunk
  uint64_t full_cols;   // columns [0, full_cols) are whole in every chunk
  uint64_t items;       // warp items of 32 / W columns
  int n;
};

// W: lanes per ring instance; NR: the rank count at compile time, or 0 for
// any count up to W (loops then run to W with a guard, so that the inputs
// stay in registers).
template <int DT, int OP, int W, int NR>
__global__ void __launch_bounds__(kRlThreads) k_ring_lane(const __grid_constant__ RingLaneArgs a) {
  using A = typename Elem<DT>::A;
  constexpr int VN = Vec<DT>::kN;  // elements per 16-byte vector
  constexpr int ES = Elem<DT>::kSize;
  constexpr int G = 32 / W;  // instances (columns) per warp
  constexpr int KMAX = NR > 0 ? NR : W;
  static_assert(NR <= W, "an instance holds every rank");
  const int n = NR > 0 ? NR : a.n;
  const int lane = static_cast<int>(threadIdx.x & 31);
  const int warp = static_cast<int>(threadIdx.x >> 5);
  const int r = lane & (W - 1);
  const int g = lane / W;
  const bool active = r < n;
  const int from = (lane & ~(W - 1)) | (r == 0 ? n - 1 : r - 1);  // the predecessor's lane
  pdl_wait();
  pdl_trigger();

  const uint64_t seg_b = a.seg * ES;
  const char* const in_r = a.in[active ? r : 0];
  char* const out_r = a.out[active ? r : 0];
  const int c0 = r == 0 ? n - 1 : r - 1;  // chunk of reduce-scatter step 0
  // the vector at column col of chunk c is inside the message
  auto inside = [&](int c, uint64_t col) {
    return static_cast<uint64_t>(c) * a.seg + (col + 1) * VN <= a.count;
  };

  uint4 x[KMAX];
  auto load = [&](uint64_t item) {
    const uint64_t col = item * G + g;
    const bool full = (item + 1) * G <= a.full_cols;
    const bool ok = active && col < a.cols;
    int c = c0;
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (k >= n) break;
      x[k] = make_uint4(0, 0, 0, 0);
      if (ok && (full || inside(c, col))) x[k] = ld16(in_r + static_cast<uint64_t>(c) * seg_b + col * 16);
      c = c == 0 ? n - 1 : c - 1;
    }
  };

  const uint64_t wstride = static_cast<uint64_t>(gridDim.x) * kRlWarps;
  uint64_t item = static_cast<uint64_t>(blockIdx.x) * kRlWarps + warp;
  if (item < a.items) load(item);
  for (; item < a.items; item += wstride) {
    const uint64_t col = item * G + g;
    const bool full = (item + 1) * G <= a.full_cols;
    const bool ok = active && col < a.cols;
    // reduce-scatter: N-1 hops of partials
    A p[VN];
    {
      Vec<DT> w;
      widen16<DT>(x[0], w);
#pragma unroll
      for (int i = 0; i < VN; ++i) p[i] = w.v[i];
    }
#pragma unroll
    for (int k = 1; k < KMAX; ++k) {
      if (k >= n) break;
#pragma unroll
      for (int i = 0; i < VN; ++i) p[i] = __shfl_sync(0xFFFFFFFFu, p[i], from);
      Vec<DT> w;
      widen16<DT>(x[k], w);
#pragma unroll
      for (int i = 0; i < VN; ++i) p[i] = op_step<OP>(p[i], w.v[i]);
    }
    // the one rounding, on rank r (its own chunk); the rounded value travels on
    Vec<DT> v;
#pragma unroll
    for (int i = 0; i < VN; ++i) v.v[i] = p[i];
    uint4 w = narrow16<DT>(v);
    // the next item's inputs, in flight during the all-gather
    if (item + wstride < a.items) load(item + wstride);
    if (ok && (full || inside(r, col))) st16(out_r + static_cast<uint64_t>(r) * seg_b + col * 16, w);
    // all-gather: N-1 hops; at hop j chunk r - j arrives and is stored
    int c = r;
#pragma unroll
    for (int j = 1; j < KMAX; ++j) {
      if (j >= n) break;
      w.x = __shfl_sync(0xFFFFFFFFu, w.x, from);
      w.y = __shfl_sync(0xFFFFFFFFu, w.y, from);
      w.z = __shfl_sync(0xFFFFFFFFu, w.z, from);
      w.w = __shfl_sync(0xFFFFFFFFu, w.w, from);
      c = c == 0 ? n - 1 : c - 1;
      if (ok && (full || inside(c, col))) st16(out_r + static_cast<uint64_t>(c) * seg_b + col * 16, w);
    }
  }
  if (blockIdx.x == 0 && warp == 0) ring_tail<DT, OP>(a, lane);
}

template <int DT, int OP, int W, int NR>
static int launch_ring_lane_t(RingLaneArgs a, cudaStream_t s) {
  constexpr int VN = Vec<DT>::kN;
  constexpr int G = 32 / W;
  a.cols = a.seg / VN;
  a.items = (a.cols + G - 1) / G;
  // the last chunk is the shortest (possibly empty): a column is whole in
  // every chunk when it is whole in that one
  const uint64_t lead = static_cast<uint64_t>(a.n - 1) * a.seg;
  a.full_cols = a.count > lead ? std::min<uint64_t>(a.cols, (a.count - lead) / VN) : 0;
  static int per_sm[COLL_MAX_RANKS] = {0};  // resident CTAs per SM, per device ordinal (benign race)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= COLL_MAX_RANKS) dev = 0;
  if (per_sm[dev] == 0) {
    int v = 0;
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, k_ring_lane<DT, OP, W, NR>, kRlThreads, 0);
    if (e != cudaSuccess || v <= 0) {
      (void)cudaGetLastError();
      return launch_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
    }
    per_sm[dev] = v;
  }
  const uint64_t need = std::max<uint64_t>(1, (a.items + kRlWarps - 1) / kRlWarps);
  const uint64_t grid = std::min<uint64_t>(need, static_cast<uint64_t>(num_sms()) * per_sm[dev]);
  launch_pdl(k_ring_lane<DT, OP, W, NR>, dim3(static_cast<unsigned>(grid)), dim3(kRlThreads), 0, s, a);
  return launch_status(cudaGetLastError());
}

template <int DT, int OP>
static int launch_ring_lane_op(const RingLaneArgs& a, cudaStream_t s) {
  switch (a.n) {
    case 2: return launch_ring_lane_t<DT, OP, 2, 2>(a, s);
    case 3: return launch_ring_lane_t<DT, OP, 4, 0>(a, s);
    case 4: return launch_ring_lane_t<DT, OP, 4, 4>(a, s);
    case 8: return launch_ring_lane_t<DT, OP, 8, 8>(a, s);
    default: return launch_ring_lane_t<DT, OP, 8, 0>(a, s);  // 5..7
  }
}

template <int DT>
static int launch_ring_lane_dt(const RingLaneArgs& a, coll_op_t op, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_ring_lane_op<DT, COLL_SUM>(a, s);
    case COLL_MAX: return launch_ring_lane_op<DT, COLL_MAX>(a, s);
    case COLL_MIN: return launch_ring_lane_op<DT, COLL_MIN>(a, s);
    case COLL_PROD: return launch_ring_lane_op<DT, COLL_PROD>(a, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

bool ring_lane_supported(int n) { return n >= 2 && n <= 8; }

int launch_ring_lane(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                     cudaStream_t s) {
  RingLaneArgs a{};
  for (int r = 0; r < n; ++r) {
    a.in[r] = in[r];
    a.out[r] = out[r];
  }
  const int es = elem_size(dt);
  const size_t g = 16 / es;
  a.seg = ((count + n - 1) / n + g - 1) / g * g;
  a.count = count;
  a.n = n;
  switch (dt) {
    case COLL_BF16: return launch_ring_lane_dt<COLL_BF16>(a, op, s);
    case COLL_FP16: return launch_ring_lane_dt<COLL_FP16>(a, op, s);
    case COLL_FP32: return launch_ring_lane_dt<COLL_FP32>(a, op, s);
    case COLL_INT32: return launch_ring_lane_dt<COLL_INT32>(a, op, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

}  // namespace mvr
