// Two-shot all-reduce in ONE cooperative launch with LL packets between the
// virtual ranks ("From NCCL Ring LL to PCIe IPC AllReduce": the LL line
// [4 B data | 4 B flag] of "Traditional LL Protocols", and the owner-segment
// two-shot scheme of the "Pro5000 ?" A/B/C/D example).
//
// Three phases, each done by every thread over its share of the 16-byte
// element groups, with no barrier between them:
//   A  rank r writes each group of its input, as LL lines, into the receive
//      area of the group's owner s (FIFO_rs[s][r]);
//   B  owner s polls FIFO_rs[s][q] for q = 0 .. N-1 until every line's flag
//      is current, adds the values in rank order in fp32 (int32 for int32),
//      rounds once and writes the result as LL lines into FIFO_ag[q][s] for
//      every rank q;
//   C  rank q polls FIFO_ag[q][s] and stores the values into its output.
// A never waits, B waits only on A and C only on B, and all CTAs are
// resident (cooperative launch), so every poll ends.  The arithmetic is that
// of coll_all_reduce(TWOSHOT): the result is bit-identical.
//
// A line's flag is (epoch << 2) | phase, where the epoch is a call counter
// in the workspace header advanced by the last CTA to finish, so lines left
// by an earlier call never match.  The epoch has 30 bits: a call that finds
// the counter at 2^30 does nothing and raises COLL_DEV_EPOCH_WRAP.  Every poll is bounded: after the budget a
// thread raises COLL_DEV_TIMEOUT and sets the header's abort word, which
// stops the other polls.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace mvr {

constexpr long long kTsllBudgetCycles = 2ll << 30;  // about 1 s at 1.9 GHz
constexpr int kTsllThreads = 256;
constexpr int kTsllBatch = 8;  // sources polled together in phase B

struct TwoShotLLArgs {
  const char* in[kMaxRanks];
  char* out[kMaxRanks];
  uint4* fifo_rs;  // [owner s][source r][seg * ES / 8] 16-byte units (2 LL lines each)
  uint4* fifo_ag;  // [rank q][owner s][seg * ES / 8]
  uint32_t* hdr;   // [0] epoch, [1] finished CTAs, [2] abort
  uint64_t count, seg;
  int n, groups;
  int* status;
};

__device__ __forceinline__ void tsll_st16(uint4* p, const uint4& v) {
  asm volatile("st.volatile.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 tsll_ld16(const uint4* p) {
  uint4 v;
  asm volatile("ld.volatile.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ uint32_t tsll_ld32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.volatile.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <int DT, int OP>
__global__ void __launch_bounds__(kTsllThreads) k_twoshot_ll(const __grid_constant__ TwoShotLLArgs a) {
  using A = typename Elem<DT>::A;
  using S = typename Elem<DT>::S;
  constexpr int VN = Vec<DT>::kN;  // elements per 16-byte group
  constexpr int ES = Elem<DT>::kSize;
  const int n = a.n;
  const int r = blockIdx.x % n;
  const int g = blockIdx.x / n;
  const uint32_t epoch = tsll_ld32(a.hdr);
  // all CTAs read the same counter (the last CTA of a call advances it after
  // every CTA has read it) and leave together: past the last epoch the flags
  // would repeat those of epoch 0
  if (epoch >= COLL_TWOSHOT_LL_CALLS_PER_FILL) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(a.status, COLL_DEV_EPOCH_WRAP, 1);
    return;
  }
  const uint32_t flag_rs = (epoch << 2) | 1u, flag_ag = (epoch << 2) | 2u;
  const uint64_t units_per_seg = a.seg * ES / 8;  // 16-byte units (8 payload bytes each) per segment
  const uint64_t first = static_cast<uint64_t>(g) * blockDim.x + threadIdx.x;
  const uint64_t stride = static_cast<uint64_t>(a.groups) * blockDim.x;
  const uint64_t ngroups = (a.count + VN - 1) / VN;  // groups of a rank's buffer
  bool alive = true;

  // 16 payload bytes -> the two units {d0, f, d1, f}, {d2, f, d3, f}
  auto pack = [](const uint4& w, uint32_t f, uint4& u0, uint4& u1) {
    u0 = make_uint4(w.x, f, w.y, f);
    u1 = make_uint4(w.z, f, w.w, f);
  };
  // poll a unit pair until all four flags equal f (bounded); false on timeout or abort
  auto poll = [&](const uint4* p, uint32_t f, uint4& u0, uint4& u1) -> bool {
    long long t0 = 0;
    for (int it = 0;; ++it) {
      const bool ok0 = u0.y == f && u0.w == f, ok1 = u1.y == f && u1.w == f;
      if (ok0 && ok1) return true;
      if (it == 0) t0 = clock64();
      if ((it & 255) == 255) {
        if (tsll_ld32(a.hdr + 2) != 0) return false;
        if (clock64() - t0 > kTsllBudgetCycles) {
          report(a.status, COLL_DEV_TIMEOUT, 1);
          atomicExch(a.hdr + 2, 1u);
          return false;
        }
      }
      if (!ok0) u0 = tsll_ld16(p);
      if (!ok1) u1 = tsll_ld16(p + 1);
    }
  };

  pdl_wait();
  // A: my input, group by group, to the group's owner
  for (uint64_t i = first; i < ngroups; i += stride) {
    const uint64_t gi = i * VN;
    union {
      uint4 u;
      S s[VN];
    } w;
    if (gi + VN <= a.count) {
      w.u = ld16(a.in[r] + gi * ES);
    } else {  // ragged tail, zero-padded
#pragma unroll
      for (int j = 0; j < VN; ++j) w.s[j] = gi + j < a.count ? *reinterpret_cast<const S*>(a.in[r] + (gi + j) * ES) : S(0);
    }
    const uint64_t s = gi / a.seg, e = gi - s * a.seg;
    uint4* p = a.fifo_rs + (s * n + r) * units_per_seg + e * ES / 8;
    uint4 u0, u1;
    pack(w.u, flag_rs, u0, u1);
    tsll_st16(p, u0);
    tsll_st16(p + 1, u1);
  }
  pdl_trigger();

  // B: I own segment r: reduce it over the ranks in rank order and send it to all
  const uint64_t seg_lo = static_cast<uint64_t>(r) * a.seg;
  const uint64_t seg_groups = a.count > seg_lo ? (min(a.seg, a.count - seg_lo) + VN - 1) / VN : 0;
  for (uint64_t i = first; alive && i < seg_groups; i += stride) {
    const uint64_t e = i * VN;
    A acc[VN];
    for (int q0 = 0; q0 < n && alive; q0 += kTsllBatch) {
      uint4 u[kTsllBatch][2];
      const uint4* p[kTsllBatch];
#pragma unroll
      for (int b = 0; b < kTsllBatch; ++b) {  // issue the batch's loads together
        p[b] = a.fifo_rs + (static_cast<uint64_t>(r) * n + q0 + b) * units_per_seg + e * ES / 8;
        if (q0 + b < n) {
          u[b][0] = tsll_ld16(p[b]);
          u[b][1] = tsll_ld16(p[b] + 1);
        }
      }
#pragma unroll
      for (int b = 0; b < kTsllBatch; ++b) {
        if (q0 + b < n && alive) {
          if (!poll(p[b], flag_rs, u[b][0], u[b][1])) {
            alive = false;
          } else {
            Vec<DT> x;
            widen16<DT>(make_uint4(u[b][0].x, u[b][0].z, u[b][1].x, u[b][1].z), x);
            if (q0 + b == 0) {
#pragma unroll
              for (int j = 0; j < VN; ++j) acc[j] = x.v[j];
            } else {
#pragma unroll
              for (int j = 0; j < VN; ++j) acc[j] = op_step<OP>(acc[j], x.v[j]);
            }
          }
        }
      }
    }
    if (!alive) break;
    Vec<DT> w;
#pragma unroll
    for (int j = 0; j < VN; ++j) w.v[j] = acc[j];
    uint4 u0, u1;
    pack(narrow16<DT>(w), flag_ag, u0, u1);
    for (int q = 0; q < n; ++q) {
      uint4* d = a.fifo_ag + (static_cast<uint64_t>(q) * n + r) * units_per_seg + e * ES / 8;
      tsll_st16(d, u0);
      tsll_st16(d + 1, u1);
    }
  }

  // C: the reduced groups of every owner into my output
  for (uint64_t i = first; alive && i < ngroups; i += stride) {
    const uint64_t gi = i * VN;
    const uint64_t s = gi / a.seg, e = gi - s * a.seg;
    const uint4* p = a.fifo_ag + (static_cast<uint64_t>(r) * n + s) * units_per_seg + e * ES / 8;
    uint4 u0 = tsll_ld16(p), u1 = tsll_ld16(p + 1);
    if (!poll(p, flag_ag, u0, u1)) {
      alive = false;
      break;
    }
    union {
      uint4 u;
      S s[VN];
    } w;
    w.u = make_uint4(u0.x, u0.z, u1.x, u1.z);
    if (gi + VN <= a.count) {
      st16(a.out[r] + gi * ES, w.u);
    } else {
#pragma unroll
      for (int j = 0; j < VN; ++j)
        if (gi + j < a.count) *reinterpret_cast<S*>(a.out[r] + (gi + j) * ES) = w.s[j];
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

size_t twoshot_ll_workspace(int n, size_t count, int es) {
  const size_t g = 16 / es;
  const size_t seg = ((count + n - 1) / n + g - 1) / g * g;
  return 256 + 2 * (2 * static_cast<size_t>(n) * n * seg * es);  // two FIFOs of N x N segments, 8 B per 4 B
}

template <int DT, int OP>
static int launch_twoshot_ll_t(TwoShotLLArgs& a, cudaStream_t s) {
  static int max_per_sm[COLL_MAX_RANKS] = {0};  // per device ordinal (benign race: same value)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= COLL_MAX_RANKS) dev = 0;
  if (max_per_sm[dev] == 0) {
    int v = 0;
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, k_twoshot_ll<DT, OP>, kTsllThreads, 0);
    if (e != cudaSuccess || v <= 0) {
      (void)cudaGetLastError();
      return launch_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
    }
    max_per_sm[dev] = v;
  }
  constexpr int VN = Vec<DT>::kN;
  const uint64_t ngroups = (a.count + VN - 1) / VN;
  const int max_groups = max_per_sm[dev] * num_sms() / a.n;
  if (max_groups < 1) return COLL_ERR_UNSUPPORTED;  // more ranks than co-resident CTAs
  a.groups = static_cast<int>(std::min<uint64_t>((ngroups + kTsllThreads - 1) / kTsllThreads, max_groups));
  if (a.groups < 1) a.groups = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(a.groups * a.n));
  cfg.blockDim = dim3(kTsllThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_twoshot_ll<DT, OP>, a);
  if (e != cudaSuccess) (void)cudaGetLastError();  // reported here; keep it from surfacing in a later call
  return launch_status(e);
}

template <int DT>
static int launch_twoshot_ll_dt(TwoShotLLArgs& a, coll_op_t op, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_twoshot_ll_t<DT, COLL_SUM>(a, s);
    case COLL_MAX: return launch_twoshot_ll_t<DT, COLL_MAX>(a, s);
    case COLL_MIN: return launch_twoshot_ll_t<DT, COLL_MIN>(a, s);
    case COLL_PROD: return launch_twoshot_ll_t<DT, COLL_PROD>(a, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

int launch_twoshot_ll(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                      void* workspace, int* status, cudaStream_t s) {
  TwoShotLLArgs a{};
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
  a.hdr = static_cast<uint32_t*>(workspace);
  a.fifo_rs = reinterpret_cast<uint4*>(static_cast<char*>(workspace) + 256);
  a.fifo_ag = a.fifo_rs + static_cast<size_t>(n) * n * a.seg * es / 8;
  switch (dt) {
    case COLL_BF16: return launch_twoshot_ll_dt<COLL_BF16>(a, op, s);
    case COLL_FP16: return launch_twoshot_ll_dt<COLL_FP16>(a, op, s);
    case COLL_FP32: return launch_twoshot_ll_dt<COLL_FP32>(a, op, s);
    case COLL_INT32: return launch_twoshot_ll_dt<COLL_INT32>(a, op, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

}  // namespace mvr
