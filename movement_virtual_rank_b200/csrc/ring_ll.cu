// Single-launch ring all-reduce with LL packets between neighbouring virtual
// ranks ("From NCCL Ring LL to PCIe IPC AllReduce", sections "Traditional LL
// Protocols" and "Pro5000 ?": the sender writes [4 B data | 4 B flag] lines
// into the receiver's FIFO with 16-byte stores, the receiver re-reads 16-byte
// groups until both flags equal the current step and only then uses the data).
//
// Virtual rank r is played by CTAs blockIdx.x = g * N + r.  Thread t of CTA
// (r, g) owns the same VN elements of every chunk for every rank, so it talks
// only to thread t of CTA (r-1, g) (its sender) and (r+1, g) (its receiver).
// Step k of rank r (the ring order of coll_all_reduce(RING)):
//   k = 0            send own chunk c = r-1 (widened) to r+1, FIFO slot 0
//   k = 1 .. N-2     receive slot k-1, add own chunk c = r-1-k, send slot k
//   k = N-1          receive slot N-2, add own chunk r: the sum is complete;
//                    round it, write it to out[r], send it on (slot N-1)
//   j = 1 .. N-1     receive slot N-2+j = finished chunk r-j, write it to
//                    out[r], forward it (slot N-1+j) unless j = N-1
// Every slot has its own FIFO space, so no line is ever overwritten while it
// may still be read, and no back-pressure is needed.  A line's flag is
// (epoch << 7) | (slot + 1), where the epoch is a per-workspace call counter
// kept in the workspace header (advanced by the last CTA to finish), so lines
// left by an earlier call never match.  The epoch has 25 bits: a call that
// finds the counter at 2^25 does nothing and raises COLL_DEV_EPOCH_WRAP.
//
// All CTAs are co-resident (cooperative launch).  Every poll is bounded: after
// the budget a CTA raises COLL_DEV_TIMEOUT, sets the header's abort word (so
// that the others stop polling) and returns; nothing can hang.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace mvr {

constexpr long long kPollBudgetCycles = 2ll << 30;  // about 1 s at 1.9 GHz
constexpr int kRingLLThreads = 256;

struct RingLLArgs {
  const char* in[kMaxRanks];
  char* out[kMaxRanks];
  uint4* fifo;       // [N receivers][2N-2 slots][seg lines] of 8 bytes, as 16-byte pairs
  uint32_t* hdr;     // [0] epoch, [1] finished CTAs, [2] abort
  uint64_t count, seg;
  int n, groups;
  int* status;
};

__device__ __forceinline__ void st_volatile16(uint4* p, const uint4& v) {
  asm volatile("st.volatile.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_volatile16(const uint4* p) {
  uint4 v;
  asm volatile("ld.volatile.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_volatile32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.volatile.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <typename A>
__device__ __forceinline__ uint32_t a_bits(A v) {
  if constexpr (std::is_same<A, float>::value) return __float_as_uint(v);
  else return static_cast<uint32_t>(v);
}
template <typename A>
__device__ __forceinline__ A bits_a(uint32_t u) {
  if constexpr (std::is_same<A, float>::value) return __uint_as_float(u);
  else return static_cast<A>(static_cast<int32_t>(u));
}

template <int DT, int OP>
__global__ void __launch_bounds__(kRingLLThreads) k_ring_ll(const __grid_constant__ RingLLArgs a) {
  using A = typename Elem<DT>::A;
  using S = typename Elem<DT>::S;
  constexpr int VN = Vec<DT>::kN;   // elements per thread = per 16-byte input group
  constexpr int NG = VN / 2;        // 16-byte line pairs per thread per slot
  constexpr int ES = Elem<DT>::kSize;
  const int n = a.n;
  const int r = blockIdx.x % n;
  const int g = blockIdx.x / n;
  const int slots = 2 * n - 2;
  const uint32_t epoch = ld_volatile32(a.hdr);
  // every CTA reads the same counter (only the last CTA of a call advances
  // it, after all have read it), so all take this exit together: past the
  // last epoch the flags would repeat those of epoch 0, and a line no call
  // has rewritten since could pass for a current one
  if (epoch >= COLL_RING_LL_CALLS_PER_FILL) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(a.status, COLL_DEV_EPOCH_WRAP, 1);
    return;
  }
  const int rs = (r + 1) % n;  // receiver of my sends
  bool alive = true;

  // FIFO of receiver q, slot s, element offset e (a multiple of VN): NG pairs of lines
  auto fifo_at = [&](int q, int s, uint64_t e) {
    return a.fifo + ((static_cast<uint64_t>(q) * slots + s) * a.seg + e) / 2;
  };
  auto flag_of = [&](int s) { return (epoch << 7) | static_cast<uint32_t>(s + 1); };

  auto send = [&](int s, uint64_t e, const A (&v)[VN]) {
    uint4* p = fifo_at(rs, s, e);
    const uint32_t f = flag_of(s);
#pragma unroll
    for (int i = 0; i < NG; ++i) st_volatile16(p + i, make_uint4(a_bits(v[2 * i]), f, a_bits(v[2 * i + 1]), f));
  };
  // wait for my sender's lines of slot s (bounded); false on timeout or abort
  auto recv = [&](int s, uint64_t e, A (&v)[VN]) -> bool {
    const uint4* p = fifo_at(r, s, e);
    const uint32_t f = flag_of(s);
    uint4 x[NG];
#pragma unroll
    for (int i = 0; i < NG; ++i) x[i] = ld_volatile16(p + i);
    long long t0 = 0;
    for (int it = 0;; ++it) {
      bool ok = true;
#pragma unroll
      for (int i = 0; i < NG; ++i) ok = ok && x[i].y == f && x[i].w == f;
      if (ok) break;
      if (it == 0) t0 = clock64();
      if ((it & 255) == 255) {
        if (ld_volatile32(a.hdr + 2) != 0) return false;  // another CTA gave up
        if (clock64() - t0 > kPollBudgetCycles) {
          report(a.status, COLL_DEV_TIMEOUT, 1);
          atomicExch(a.hdr + 2, 1u);
          return false;
        }
      }
#pragma unroll
      for (int i = 0; i < NG; ++i)
        if (!(x[i].y == f && x[i].w == f)) x[i] = ld_volatile16(p + i);
    }
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      v[2 * i] = bits_a<A>(x[i].x);
      v[2 * i + 1] = bits_a<A>(x[i].z);
    }
    return true;
  };
  // my rank's input values of chunk c at element offset e (zero past the end)
  auto own = [&](int c, uint64_t e, A (&v)[VN]) {
    const uint64_t lo = static_cast<uint64_t>(c) * a.seg;
    const uint64_t gi = lo + e;
    const uint64_t end = min(lo + a.seg, a.count);
    if (gi + VN <= end) {
      Vec<DT> w;
      widen16<DT>(ld16(a.in[r] + gi * ES), w);
#pragma unroll
      for (int i = 0; i < VN; ++i) v[i] = w.v[i];
    } else {
#pragma unroll
      for (int i = 0; i < VN; ++i)
        v[i] = gi + i < end ? widen1<DT>(*reinterpret_cast<const S*>(a.in[r] + (gi + i) * ES)) : A(0);
    }
  };
  auto put = [&](int c, uint64_t e, const A (&v)[VN]) {
    const uint64_t lo = static_cast<uint64_t>(c) * a.seg;
    const uint64_t gi = lo + e;
    const uint64_t end = min(lo + a.seg, a.count);
    if (gi + VN <= end) {
      Vec<DT> w;
#pragma unroll
      for (int i = 0; i < VN; ++i) w.v[i] = v[i];
      st16(a.out[r] + gi * ES, narrow16<DT>(w));
    } else {
#pragma unroll
      for (int i = 0; i < VN; ++i)
        if (gi + i < end) *reinterpret_cast<S*>(a.out[r] + (gi + i) * ES) = narrow1<DT>(v[i]);
    }
  };

  // The rank's own inputs are final before the kernel starts, so the values
  // it adds at the first kPreload reduce-scatter steps are fetched up front:
  // each hop then costs only the LL hand-off, not an extra trip to DRAM after
  // the poll succeeds.  (The steps are unrolled so the values stay in
  // registers.)
  constexpr int kPreload = 8;
  const uint64_t stride = static_cast<uint64_t>(a.groups) * blockDim.x * VN;
  for (uint64_t e = (static_cast<uint64_t>(g) * blockDim.x + threadIdx.x) * VN; alive && e < a.seg; e += stride) {
    A p[VN];
    uint4 pre[kPreload];
#pragma unroll
    for (int k = 0; k < kPreload; ++k) {
      pre[k] = make_uint4(0, 0, 0, 0);
      if (k < n) {
        const int c = ((r - 1 - k) % n + n) % n;
        const uint64_t gi = static_cast<uint64_t>(c) * a.seg + e;
        const uint64_t end = min(static_cast<uint64_t>(c) * a.seg + a.seg, a.count);
        if (gi + VN <= end) pre[k] = ld16(a.in[r] + gi * ES);
      }
    }
    // the values rank r adds at step k (chunk c): preloaded, or read now
    auto own_at = [&](const uint4& v, int c, A (&out)[VN]) {
      const uint64_t gi = static_cast<uint64_t>(c) * a.seg + e;
      const uint64_t end = min(static_cast<uint64_t>(c) * a.seg + a.seg, a.count);
      if (gi + VN <= end) {
        Vec<DT> w;
        widen16<DT>(v, w);
#pragma unroll
        for (int i = 0; i < VN; ++i) out[i] = w.v[i];
      } else {
        own(c, e, out);
      }
    };
    // one reduce-scatter step k >= 1: receive, add my values, (round,) send
    auto rs_step = [&](int k, const A (&xv)[VN]) -> bool {
      if (!recv(k - 1, e, p)) return false;
#pragma unroll
      for (int i = 0; i < VN; ++i) p[i] = op_step<OP>(p[i], xv[i]);
      if (k == n - 1) {
        // complete on rank r: round once; what travels on is the rounded value
        Vec<DT> w;
#pragma unroll
        for (int i = 0; i < VN; ++i) w.v[i] = p[i];
        Vec<DT> back;
        widen16<DT>(narrow16<DT>(w), back);
#pragma unroll
        for (int i = 0; i < VN; ++i) p[i] = back.v[i];
        put(r, e, p);
      }
      send(k, e, p);
      return true;
    };
    // reduce-scatter phase
    own_at(pre[0], (r - 1 + n) % n, p);
    send(0, e, p);
#pragma unroll
    for (int k = 1; k < kPreload; ++k) {
      if (k >= n || !alive) break;
      A xv[VN];
      own_at(pre[k], ((r - 1 - k) % n + n) % n, xv);
      alive = rs_step(k, xv);
    }
    for (int k = kPreload; k < n && alive; ++k) {
      A xv[VN];
      own(((r - 1 - k) % n + n) % n, e, xv);
      alive = rs_step(k, xv);
    }
    // all-gather phase
    for (int j = 1; j < n && alive; ++j) {
      if (!recv(n - 2 + j, e, p)) {
        alive = false;
        break;
      }
      put(((r - j) % n + n) % n, e, p);
      if (j < n - 1) send(n - 1 + j, e, p);
    }
  }
  // the last CTA to finish advances the epoch and clears the abort word
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t done = atomicAdd(a.hdr + 1, 1u);
    if (done == gridDim.x - 1) {
      atomicExch(a.hdr + 1, 0u);
      atomicExch(a.hdr + 2, 0u);
      atomicExch(a.hdr, epoch + 1);
    }
  }
}

// one thread re-reads *flag until it equals `expect`, bounded by budget_us of
// %globaltimer time; raises COLL_DEV_TIMEOUT when the budget runs out
__global__ void k_wait_flag(const uint32_t* flag, uint32_t expect, uint64_t budget_ns, int* status) {
  pdl_wait();
  pdl_trigger();
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (;;) {
    if (ld_volatile32(flag) == expect) return;
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > budget_ns) {
      report(status, COLL_DEV_TIMEOUT, 1);
      return;
    }
    __nanosleep(1000);
  }
}

int launch_wait_flag(const uint32_t* flag, uint32_t expect, uint32_t budget_us, int* status, cudaStream_t s) {
  launch_pdl(k_wait_flag, dim3(1), dim3(1), 0, s, flag, expect, static_cast<uint64_t>(budget_us) * 1000ull, status);
  return launch_status(cudaGetLastError());
}

size_t ring_ll_workspace(int n, size_t count, int es) {
  const size_t g = 16 / es;
  const size_t seg = ((count + n - 1) / n + g - 1) / g * g;
  const size_t slots = n > 1 ? 2 * static_cast<size_t>(n) - 2 : 0;
  return 256 + static_cast<size_t>(n) * slots * seg * 8;
}

template <int DT, int OP>
static int launch_ring_ll_t(RingLLArgs& a, cudaStream_t s) {
  static int max_per_sm[COLL_MAX_RANKS] = {0};  // per device ordinal (benign race: same value)
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= COLL_MAX_RANKS) dev = 0;
  if (max_per_sm[dev] == 0) {
    int v = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, k_ring_ll<DT, OP>, kRingLLThreads, 0);
    if (e != cudaSuccess || v <= 0) return launch_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
    max_per_sm[dev] = v;
  }
  constexpr int VN = Vec<DT>::kN;
  const uint64_t per_group = static_cast<uint64_t>(kRingLLThreads) * VN;
  const int max_groups = std::max(1, max_per_sm[dev] * num_sms() / a.n);
  a.groups = static_cast<int>(std::min<uint64_t>((a.seg + per_group - 1) / per_group, max_groups));
  if (a.groups < 1) a.groups = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(a.groups * a.n));
  cfg.blockDim = dim3(kRingLLThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return launch_status(cudaLaunchKernelEx(&cfg, k_ring_ll<DT, OP>, a));
}

template <int DT>
static int launch_ring_ll_dt(RingLLArgs& a, coll_op_t op, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_ring_ll_t<DT, COLL_SUM>(a, s);
    case COLL_MAX: return launch_ring_ll_t<DT, COLL_MAX>(a, s);
    case COLL_MIN: return launch_ring_ll_t<DT, COLL_MIN>(a, s);
    case COLL_PROD: return launch_ring_ll_t<DT, COLL_PROD>(a, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

int launch_ring_ll(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                   void* workspace, int* status, cudaStream_t s) {
  RingLLArgs a{};
  for (int r = 0; r < n; ++r) {
    a.in[r] = in[r];
    a.out[r] = out[r];
  }
  const int es = elem_size(dt);
  const size_t g = 16 / es;
  a.seg = ((count + n - 1) / n + g - 1) / g * g;
  a.count = count;
  a.n = n;
  a.hdr = static_cast<uint32_t*>(workspace);
  a.fifo = reinterpret_cast<uint4*>(static_cast<char*>(workspace) + 256);
  a.status = status;
  switch (dt) {
    case COLL_BF16: return launch_ring_ll_dt<COLL_BF16>(a, op, s);
    case COLL_FP16: return launch_ring_ll_dt<COLL_FP16>(a, op, s);
    case COLL_FP32: return launch_ring_ll_dt<COLL_FP32>(a, op, s);
    case COLL_INT32: return launch_ring_ll_dt<COLL_INT32>(a, op, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

}  // namespace mvr
