// Ring all-reduce with the virtual ranks as the CTAs of one thread-block
// cluster: the hop from rank r to rank r+1 goes over distributed shared
// memory (the SM-to-SM network), not through HBM or a kernel boundary.
//
// The schedule, chunk order, fp32 partials and the single rounding are those
// of coll_all_reduce(RING) (TP communication essay; NCCL's ring kernel named
// in "From NCCL Ring LL to PCIe IPC AllReduce"), so the result is
// bit-identical.  CTA r of a cluster of N plays virtual rank r; the segment
// is cut into tiles of TH x VN elements per chunk (TH = 64 threads per CTA for
// most messages up to 512 KB per rank, whose hops then carry fewer bytes and
// land sooner; 128 above), and the clusters
// walk the tiles with a stride (persistent: about as many clusters as fit on
// the GPU at once).  Thread t owns VN elements of each chunk of a tile.
//
// Hop transport.  For each of the 2N-2 hops of a tile the sender stores its
// values straight into a slot of the receiver's shared memory with
// st.async ... mbarrier::complete_tx, so the store itself completes the
// receiver's mbarrier for that slot (release at cluster scope, no separate
// fence or arrive).  The receiver armed that mbarrier with the slot's byte
// count and waits on it (acquire at cluster scope).  Hops are numbered
// without a break from tile to tile and hop h uses slot h mod N: the ring's
// own dependencies keep a sender within N-1 hops of its receiver, so N slots
// per CTA are enough and need neither credits nor a barrier between tiles.
//
// All of a ring's dependencies stay inside one cluster, whose CTAs the
// hardware schedules together, so clusters may run in any order and in
// waves.  Every wait is bounded: a CTA whose wait runs out raises
// COLL_DEV_TIMEOUT and sets an abort word in every CTA of its cluster; all
// of them stop sending and receiving, meet at the final cluster barrier, and
// before leaving poll (bounded) the slots they still expect, so that no
// store is in flight into a CTA that has left.  Only st.async stores and
// mbarrier updates cross CTAs; there is no bulk copy and no multicast.
#include <algorithm>

#include "bulk.cuh"
#include "common.cuh"
#include "internal.h"

namespace mvr {

constexpr size_t kRcSmallBytes = 512 * 1024;  // per rank: 64-thread CTAs up to here, 128 above
constexpr int kRcMaxRanks = 8;                    // portable cluster size
constexpr long long kRcBudgetCycles = 1ll << 28;  // about 0.14 s per wait
constexpr long long kRcDrainCycles = 1ll << 17;   // about 70 us per slot, abort path only

struct RingClusterArgs {
  const char* in[kMaxRanks];
  char* out[kMaxRanks];
  uint64_t count, seg, tiles;
  int n;
  int* status;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_idx() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
// shared::cluster address of my shared variable at `p` in CTA `rank`
__device__ __forceinline__ uint32_t map_to(const void* p, uint32_t rank) {
  uint32_t local = static_cast<uint32_t>(__cvta_generic_to_shared(p)), remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  return remote;
}
// 16 bytes into another CTA's shared memory, completing 16 bytes of the
// transaction count of that CTA's mbarrier at `bar_addr`
__device__ __forceinline__ void st_async16(uint32_t addr, const uint4& v, uint32_t bar_addr) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
      "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(bar_addr)
      : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_volatile_smem(const uint32_t* p) {
  return *reinterpret_cast<const volatile uint32_t*>(p);
}
__device__ __forceinline__ bool try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar))), "r"(parity)
      : "memory");
  return ok != 0;
}

template <int DT, int OP, int TH>
__global__ void __launch_bounds__(TH) k_ring_cluster(const __grid_constant__ RingClusterArgs a) {
  using A = typename Elem<DT>::A;
  using S = typename Elem<DT>::S;
  constexpr int VN = Vec<DT>::kN;  // elements per thread (16 bytes of input)
  constexpr int NQ = VN / 4;       // 16-byte pieces of fp32 / int32 partials per thread
  constexpr int ES = Elem<DT>::kSize;
  constexpr uint64_t TE = static_cast<uint64_t>(TH) * VN;  // elements of a chunk per tile
  // reduce-scatter hops carry fp32 / int32 partials, all-gather hops the
  // rounded values in the storage type (16 bytes per thread)
  constexpr uint32_t kWideBytes = TH * NQ * 16;
  constexpr uint32_t kNarrowBytes = TH * 16;
  constexpr uint32_t kSlotU4 = TH * NQ;  // slot size in 16-byte units
  extern __shared__ __align__(16) uint4 slot_buf[];  // [slot][kSlotU4]
  __shared__ __align__(8) uint64_t bar[kRcMaxRanks];
  __shared__ uint32_t abort_word;
  const int n = a.n;
  const uint32_t H = 2 * n - 2;  // hops per tile: n-1 reduce-scatter, then n-1 all-gather
  const int r = static_cast<int>(cluster_rank());
  const uint64_t g = cluster_idx();
  const uint64_t G = cluster_count();
  const int tid = threadIdx.x;
  // hop h of this cluster (tile after tile) lands in slot h % n, phase h / n
  const uint32_t total_hops = static_cast<uint32_t>((a.tiles - g + G - 1) / G) * H;
  auto hop_bytes = [&](uint32_t k) { return k < static_cast<uint32_t>(n - 1) ? kWideBytes : kNarrowBytes; };
  // thread 0's record of the slots armed and not yet seen complete, and the
  // parity each was last armed for (bit j); read only by the abort drain
  uint32_t pending = 0, pending_par = 0;
  if (tid == 0) {
    abort_word = 0;
    for (int j = 0; j < n; ++j) mbar_init(&bar[j], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int j = 0; j < n; ++j) mbar_arrive_expect_tx(&bar[j], hop_bytes(j));
    pending = (1u << n) - 1;
  }
  cluster_sync_all();  // every CTA's barriers are armed before anyone stores into them
  pdl_wait();
  pdl_trigger();

  const int nxt = (r + 1) % n;
  const uint32_t next_slot0 = map_to(slot_buf, nxt);
  const uint32_t next_bar0 = map_to(bar, nxt);
  bool alive = true;

  auto chunk_lo = [&](int c) { return static_cast<uint64_t>(c) * a.seg; };
  auto chunk_end = [&](int c) { return min(chunk_lo(c) + a.seg, a.count); };
  auto to_bits = [](A x) -> uint32_t {
    if constexpr (std::is_same<A, float>::value) return __float_as_uint(x);
    else return static_cast<uint32_t>(x);
  };
  auto from_bits = [](uint32_t u) -> A {
    if constexpr (std::is_same<A, float>::value) return __uint_as_float(u);
    else return static_cast<A>(static_cast<int32_t>(u));
  };
  // store a rounded 16-byte vector (storage type) of chunk c to my output
  auto put = [&](int c, uint64_t e, const uint4& w) {
    const uint64_t gi = chunk_lo(c) + e;
    const uint64_t end = chunk_end(c);
    if (gi + VN <= end) {
      st16(a.out[r] + gi * ES, w);
    } else {
      const S* sv = reinterpret_cast<const S*>(&w);
#pragma unroll
      for (int i = 0; i < VN; ++i)
        if (gi + i < end) *reinterpret_cast<S*>(a.out[r] + (gi + i) * ES) = sv[i];
    }
  };

  // Hops are sent and received in the same order 0, 1, 2, ...: the send side
  // keeps its slot, the receive side its slot, phase parity and in-tile index.
  uint32_t js = 0;                          // slot of the next hop to send
  uint32_t hr = 0, jr = 0, pr = 0, kr = 0;  // next hop to receive: index, slot, parity, index in tile
  auto send_wide = [&](const A (&v)[VN]) {
    const uint32_t base = next_slot0 + (js * kSlotU4 + tid * NQ) * 16;
    const uint32_t bar_addr = next_bar0 + js * 8;
#pragma unroll
    for (int q = 0; q < NQ; ++q)
      st_async16(base + q * 16,
                 make_uint4(to_bits(v[4 * q]), to_bits(v[4 * q + 1]), to_bits(v[4 * q + 2]), to_bits(v[4 * q + 3])),
                 bar_addr);
    js = js + 1 == static_cast<uint32_t>(n) ? 0 : js + 1;
  };
  auto send_narrow = [&](const uint4& w) {
    st_async16(next_slot0 + (js * kSlotU4 + tid) * 16, w, next_bar0 + js * 8);
    js = js + 1 == static_cast<uint32_t>(n) ? 0 : js + 1;
  };
  // wait for the next hop; thread 0 then re-arms its slot for hop + n
  auto wait_next = [&]() -> bool {
    if (!try_wait_cluster(&bar[jr], pr)) {
      const long long t0 = clock64();
      while (!try_wait_cluster(&bar[jr], pr)) {
        if (ld_volatile_smem(&abort_word) != 0) return false;
        if (clock64() - t0 > kRcBudgetCycles) {
          report(a.status, COLL_DEV_TIMEOUT, 1);
          for (int q = 0; q < n; ++q) st_cluster_u32(map_to(&abort_word, q), 1u);
          return false;
        }
      }
    }
    return true;
  };
  auto advance = [&]() {
    if (tid == 0) {
      pending &= ~(1u << jr);
      if (hr + n < total_hops) {
        uint32_t k2 = kr + n;
        if (k2 >= H) k2 -= H;
        mbar_arrive_expect_tx(&bar[jr], hop_bytes(k2));
        pending |= 1u << jr;
        pending_par ^= 1u << jr;
      }
    }
    ++hr;
    kr = kr + 1 == H ? 0 : kr + 1;
    if (++jr == static_cast<uint32_t>(n)) {
      jr = 0;
      pr ^= 1;
    }
  };
  auto recv_wide = [&](A (&v)[VN]) -> bool {
    if (!wait_next()) return false;
    const uint4* p = slot_buf + jr * kSlotU4 + tid * NQ;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const uint4 x = p[q];
      v[4 * q] = from_bits(x.x);
      v[4 * q + 1] = from_bits(x.y);
      v[4 * q + 2] = from_bits(x.z);
      v[4 * q + 3] = from_bits(x.w);
    }
    advance();
    return true;
  };
  auto recv_narrow = [&](uint4& w) -> bool {
    if (!wait_next()) return false;
    w = slot_buf[jr * kSlotU4 + tid];
    advance();
    return true;
  };
  // the 16-byte input vectors this rank adds at each reduce-scatter step of tile t
  auto fetch = [&](uint64_t t, uint4 (&dst)[kRcMaxRanks]) {
    const uint64_t e = t * TE + static_cast<uint64_t>(tid) * VN;
#pragma unroll
    for (int k = 0; k < kRcMaxRanks; ++k) {
      dst[k] = make_uint4(0, 0, 0, 0);
      if (k < n) {
        const int c = ((r - 1 - k) % n + n) % n;
        const uint64_t gi = chunk_lo(c) + e;
        if (gi + VN <= chunk_end(c)) dst[k] = ld16(a.in[r] + gi * ES);
      }
    }
  };

  // A slot is refilled only after its previous hop was read: the sender's
  // hop h depends, thread by thread, on this rank's hop h - n + 1, which this
  // rank sends only after reading hop h - n.  So n slots need no credits.
  uint4 pre[kRcMaxRanks];
  fetch(g, pre);
  const int c0 = r == 0 ? n - 1 : r - 1;  // chunk of reduce-scatter step 0
  for (uint64_t t = g; t < a.tiles && alive; t += G) {
    const uint64_t e = t * TE + static_cast<uint64_t>(tid) * VN;
    uint4 nx[kRcMaxRanks];
    if (t + G < a.tiles) fetch(t + G, nx);  // next tile's inputs, in flight during this one
    else
#pragma unroll
      for (int k = 0; k < kRcMaxRanks; ++k) nx[k] = make_uint4(0, 0, 0, 0);

    // my values for reduce-scatter step k, chunk c (vector, or ragged tail)
    auto mine = [&](int k, int c, A (&v)[VN]) {
      const uint64_t gi = chunk_lo(c) + e;
      const uint64_t end = chunk_end(c);
      if (gi + VN <= end) {
        Vec<DT> w;
        widen16<DT>(pre[k], w);
#pragma unroll
        for (int i = 0; i < VN; ++i) v[i] = w.v[i];
      } else {
#pragma unroll
        for (int i = 0; i < VN; ++i)
          v[i] = gi + i < end ? widen1<DT>(*reinterpret_cast<const S*>(a.in[r] + (gi + i) * ES)) : A(0);
      }
    };

    A p[VN];
    int c = c0;
    mine(0, c, p);
    send_wide(p);
#pragma unroll
    for (int k = 1; k < kRcMaxRanks; ++k) {
      if (k >= n) break;
      c = c == 0 ? n - 1 : c - 1;
      A x[VN];
      mine(k, c, x);
      if (!recv_wide(p)) {
        alive = false;
        break;
      }
#pragma unroll
      for (int i = 0; i < VN; ++i) p[i] = op_step<OP>(p[i], x[i]);
      if (k < n - 1) {
        send_wide(p);
      } else {  // complete on this rank (c == r): one rounding; the rounded value travels on
        Vec<DT> w;
#pragma unroll
        for (int i = 0; i < VN; ++i) w.v[i] = p[i];
        const uint4 fin = narrow16<DT>(w);
        put(r, e, fin);
        send_narrow(fin);
      }
    }
    int cj = r;
    for (int j = 1; j < n && alive; ++j) {  // all-gather hops: chunk r - j arrives, is stored and passed on
      uint4 w;
      if (!recv_narrow(w)) {
        alive = false;
        break;
      }
      cj = cj == 0 ? n - 1 : cj - 1;
      put(cj, e, w);
      if (j < n - 1) send_narrow(w);
    }
#pragma unroll
    for (int k = 0; k < kRcMaxRanks; ++k) pre[k] = nx[k];
  }
  cluster_sync_all();  // no CTA leaves while a neighbour may still store into it
  if (tid == 0 && ld_volatile_smem(&abort_word) != 0) {
    // abort path: let any store still in flight into this CTA land first
    for (int j = 0; j < n; ++j)
      if (pending & (1u << j)) {
        const long long t0 = clock64();
        while (!try_wait_cluster(&bar[j], (pending_par >> j) & 1u) && clock64() - t0 < kRcDrainCycles) {
        }
      }
  }
}

// clusters of n CTAs that fit on the device at once (cached per device and n)
template <int DT, int OP, int TH>
static uint64_t resident_clusters(int n, size_t smem, int dev) {
  static int cache[COLL_MAX_RANKS][kRcMaxRanks + 1] = {};
  const bool cached = dev >= 0 && dev < COLL_MAX_RANKS;
  if (cached && cache[dev][n] > 0) return static_cast<uint64_t>(cache[dev][n]);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(n));
  cfg.blockDim = dim3(TH);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(n);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int v = 0;
  if (cudaOccupancyMaxActiveClusters(&v, k_ring_cluster<DT, OP, TH>, &cfg) != cudaSuccess || v <= 0) {
    (void)cudaGetLastError();
    v = std::max(1, num_sms() / n);
  }
  if (cached) cache[dev][n] = v;
  return static_cast<uint64_t>(v);
}

template <int DT, int OP, int TH>
static int launch_ring_cluster_t(RingClusterArgs a, cudaStream_t s) {
  constexpr int VN = Vec<DT>::kN;
  const uint64_t per_tile = static_cast<uint64_t>(TH) * VN;
  a.tiles = std::max<uint64_t>(1, (a.seg + per_tile - 1) / per_tile);
  const size_t smem = static_cast<size_t>(a.n) * TH * VN * 4;
  static int smem_set[COLL_MAX_RANKS] = {0};  // per device ordinal: largest limit set so far
  const int st = allow_dynamic_smem(reinterpret_cast<const void*>(k_ring_cluster<DT, OP, TH>), smem, smem_set);
  if (st != COLL_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  static bool carveout_set[COLL_MAX_RANKS] = {};  // as many CTAs per SM as shared memory allows
  if (dev >= 0 && dev < COLL_MAX_RANKS && !carveout_set[dev]) {
    if (cudaFuncSetAttribute(k_ring_cluster<DT, OP, TH>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      (void)cudaGetLastError();  // a preference only
    carveout_set[dev] = true;
  }
  const uint64_t clusters = std::min<uint64_t>(a.tiles, resident_clusters<DT, OP, TH>(a.n, smem, dev));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(clusters * a.n));
  cfg.blockDim = dim3(TH);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(a.n);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_ring_cluster<DT, OP, TH>, a);
  if (e != cudaSuccess) (void)cudaGetLastError();  // reported here; keep it from surfacing in a later call
  return launch_status(e);
}

template <int DT, int TH>
static int launch_ring_cluster_op(const RingClusterArgs& a, coll_op_t op, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_ring_cluster_t<DT, COLL_SUM, TH>(a, s);
    case COLL_MAX: return launch_ring_cluster_t<DT, COLL_MAX, TH>(a, s);
    case COLL_MIN: return launch_ring_cluster_t<DT, COLL_MIN, TH>(a, s);
    case COLL_PROD: return launch_ring_cluster_t<DT, COLL_PROD, TH>(a, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

template <int DT>
static int launch_ring_cluster_dt(const RingClusterArgs& a, coll_op_t op, cudaStream_t s) {
  // 64-thread CTAs for small messages, except where a chunk fits one 128-thread
  // tile but not one 64-thread tile: one cluster then measured faster than two
  constexpr uint64_t VN = Vec<DT>::kN;
  const bool one_wide_tile = a.seg > 64 * VN && a.seg <= 128 * VN;
  if (a.count * Elem<DT>::kSize <= kRcSmallBytes && !one_wide_tile) return launch_ring_cluster_op<DT, 64>(a, op, s);
  return launch_ring_cluster_op<DT, 128>(a, op, s);
}

bool ring_cluster_supported(int n) { return n >= 2 && n <= kRcMaxRanks; }

int launch_ring_cluster(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                        int* status, cudaStream_t s) {
  RingClusterArgs a{};
  for (int r = 0; r < n; ++r) {
    a.in[r] = in[r];
    a.out[r] = out[r];
  }
  const int es = elem_size(dt);
  const size_t g = 16 / es;
  a.seg = ((count + n - 1) / n + g - 1) / g * g;
  a.count = count;
  a.n = n;
  a.status = status;
  switch (dt) {
    case COLL_BF16: return launch_ring_cluster_dt<COLL_BF16>(a, op, s);
    case COLL_FP16: return launch_ring_cluster_dt<COLL_FP16>(a, op, s);
    case COLL_FP32: return launch_ring_cluster_dt<COLL_FP32>(a, op, s);
    case COLL_INT32: return launch_ring_cluster_dt<COLL_INT32>(a, op, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

}  // namespace mvr
