// Two-shot all-reduce in ONE cooperative launch with LL128 lines between the
// virtual ranks ("From NCCL Ring LL to PCIe IPC AllReduce": the LL128 line
// [120 B data | 8 B flag] of "Traditional LL Protocols", and the
// owner-segment two-shot scheme of the "Pro5000 ?" A/B/C/D example).
//
// The same three phases as the LL form (twoshot_ll.cu), each done by every
// warp over its share of line groups:
//   A  rank r writes each segment s of its input, as LL128 lines, into the
//      receive area of owner s (FIFO_rs[s][r]);
//   B  owner s waits for the lines of every rank, adds them in rank order in
//      fp32 (int32 for int32), rounds once and writes the result as lines
//      into FIFO_ag[q][s] for every rank q;
//   C  rank q waits for those lines and stores the values into its output.
// A never waits, B waits only on A and C only on B, and all CTAs are
// resident (cooperative launch), so every wait ends.  The arithmetic is that
// of coll_all_reduce(TWOSHOT): the result is bit-identical.
//
// Lines and their order.  A warp moves a group of 4 lines (480 payload
// bytes, 512 line bytes); lane 8l + j owns bytes [16j, 16j+16) of line l,
// lane j = 7 the line's last 8 data bytes and its 8-byte flag.  The page's
// receiver trusts a 128-byte line once its flag is current, which relies on
// the line arriving whole; on one GPU nothing makes the 8 lanes' stores of a
// line land together, so the order is made explicit: every lane stores its
// data, the warp synchronises, the flag lane fences (fence.acq_rel.gpu) and
// only then stores the flag; a reader's flag lanes poll the flags, fence,
// the warp synchronises, and only then do the lanes read their data.  An owner
// writing one group to every rank stores all the data, fences once and then
// stores all the flags; reading one group from every rank, it polls all the
// flags, fences once and then reads all the data.  Message
// offsets of a group are 16-byte aligned (480 = 30 x 16), so the message
// side moves 16-byte vectors and the bytes are rearranged in a per-warp
// shared-memory buffer.
//
// A flag is (epoch << 2) | phase in 64 bits, the epoch being the workspace's
// call counter (as in the LL form, advanced by the last CTA to finish).
// Every poll is bounded: after the budget the warp raises COLL_DEV_TIMEOUT
// and sets the header's abort word, which stops the other polls.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace mvr {

constexpr long long kT128BudgetCycles = 2ll << 30;  // about 1 s at 1.9 GHz
constexpr int kT128Threads = 256;
constexpr int kT128Warps = kT128Threads / 32;
constexpr uint64_t kGroupData = 480;  // payload bytes of a group of 4 lines
constexpr uint64_t kGroupLines = 512;

struct TwoShotLL128Args {
  const char* in[kMaxRanks];
  char* out[kMaxRanks];
  char* fifo_rs;  // [owner s][source r][gps groups][512 B]
  char* fifo_ag;  // [rank q][owner s][gps groups][512 B]
  uint32_t* hdr;  // [0] epoch, [1] finished CTAs, [2] abort
  uint64_t count, seg;  // elements of a rank's buffer, of a segment
  uint64_t gps;         // line groups per segment
  int n, groups;        // ranks, CTAs per rank
  int* status;
};

__device__ __forceinline__ void t128_st16(char* p, const uint4& v) {
  asm volatile("st.volatile.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void t128_st8(char* p, uint32_t x, uint32_t y) {
  asm volatile("st.volatile.global.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(x), "r"(y) : "memory");
}
// flags: strong (relaxed, gpu scope) stores and loads, ordered against the
// data by fence.acq_rel.gpu on the flag lane (the release and acquire
// patterns of the PTX memory model; a warp barrier carries the order to and
// from the lanes that move the data)
__device__ __forceinline__ void t128_st64(char* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void t128_fence() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ uint4 t128_ld16(const char* p) {
  uint4 v;
  asm volatile("ld.volatile.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ uint2 t128_ld8(const char* p) {
  uint2 v;
  asm volatile("ld.volatile.global.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t t128_ld64(const char* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t t128_ld32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.volatile.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <int DT, int OP>
__global__ void __launch_bounds__(kT128Threads) k_twoshot_ll128(const __grid_constant__ TwoShotLL128Args a) {
  using A = typename Elem<DT>::A;
  using S = typename Elem<DT>::S;
  constexpr int VN = Vec<DT>::kN;  // elements per 16 bytes
  constexpr int ES = Elem<DT>::kSize;
  __shared__ __align__(16) unsigned char stage[kT128Warps][kGroupData];
  const int n = a.n;
  const int r = blockIdx.x % n;
  const int g = blockIdx.x / n;
  const int warp = static_cast<int>(threadIdx.x >> 5);
  const int lane = static_cast<int>(threadIdx.x & 31);
  const int l = lane >> 3, j = lane & 7;  // line of the group, 16-byte chunk of the line
  const uint32_t epoch = t128_ld32(a.hdr);
  // every CTA reads the same counter (only the last CTA of a call advances
  // it, after all have read it), so all leave together
  if (epoch >= COLL_TWOSHOT_LL_CALLS_PER_FILL) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(a.status, COLL_DEV_EPOCH_WRAP, 1);
    return;
  }
  const uint64_t flag_rs = (static_cast<uint64_t>(epoch) << 2) | 1u;
  const uint64_t flag_ag = (static_cast<uint64_t>(epoch) << 2) | 2u;
  const uint64_t wid = static_cast<uint64_t>(g) * kT128Warps + warp;  // this warp among rank r's
  const uint64_t wstride = static_cast<uint64_t>(a.groups) * kT128Warps;
  const uint64_t seg_b = a.seg * ES;
  const uint64_t items = static_cast<uint64_t>(n) * a.gps;  // (segment, group) pairs of one rank
  unsigned char* const st = stage[warp];
  const int cpos = 120 * l + 16 * j;  // this lane's payload bytes within the group
  bool alive = true;

  // data bytes of segment s (the rest of its last group is zero padding)
  auto valid_b = [&](uint64_t s) -> uint64_t {
    const uint64_t lo = s * a.seg;
    return a.count > lo ? min(a.seg, a.count - lo) * ES : 0;
  };
  // store this lane's part of a group of lines: data first, the flag last
  auto put_group = [&](char* grp, const uint4& v, uint64_t flag) {
    char* p = grp + 128 * l + 16 * j;
    if (j < 7) t128_st16(p, v);
    else t128_st8(p, v.x, v.y);
    __syncwarp();
    if (j == 7) {
      t128_fence();
      t128_st64(p + 8, flag);
    }
  };
  // wait until the group's four flags equal `flag` (bounded); false on
  // timeout or abort (the same on every lane).  The data may be read only
  // after a fence and a warp synchronisation (read_data).
  auto wait_group = [&](const char* grp, uint64_t flag) -> bool {
    const char* p = grp + 128 * l + 16 * j;
    bool ok = j != 7;
    long long t0 = 0;
    for (int it = 0;; ++it) {
      if (!ok) ok = t128_ld64(p + 8) == flag;
      if (__all_sync(0xFFFFFFFFu, ok)) break;
      if (it == 0) t0 = clock64();
      if ((it & 255) == 255) {
        int stop = 0;
        if (lane == 0) {
          if (t128_ld32(a.hdr + 2) != 0) {
            stop = 1;  // another warp gave up
          } else if (clock64() - t0 > kT128BudgetCycles) {
            report(a.status, COLL_DEV_TIMEOUT, 1);
            atomicExch(a.hdr + 2, 1u);
            stop = 1;
          }
        }
        if (__shfl_sync(0xFFFFFFFFu, stop, 0)) return false;
      }
    }
    return true;
  };
  auto read_data = [&](const char* grp) -> uint4 {
    const char* p = grp + 128 * l + 16 * j;
    if (j < 7) return t128_ld16(p);
    const uint2 d = t128_ld8(p);
    return make_uint4(d.x, d.y, 0, 0);
  };
  auto acquire = [&]() {  // after the flags: their writers' data is visible to the whole warp
    if (j == 7) t128_fence();
    __syncwarp();
  };

  pdl_wait();
  // A: my input, segment by segment, to each segment's owner
  for (uint64_t it = wid; it < items; it += wstride) {
    const uint64_t s = it / a.gps, gi = it - s * a.gps;
    const uint64_t valid = valid_b(s);
    if (lane < 30) {
      const uint64_t o = gi * kGroupData + 16 * lane;  // byte offset within the segment
      const char* src = a.in[r] + s * seg_b + o;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (o + 16 <= valid) {
        v = ld16(src);
      } else if (o < valid) {  // the message's ragged end, element by element
        uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < VN; ++i)
          if (o + (i + 1) * ES <= valid)
            w[i * ES / 4] |= static_cast<uint32_t>(*reinterpret_cast<const S*>(src + i * ES)) << (8 * (i * ES % 4));
        v = make_uint4(w[0], w[1], w[2], w[3]);
      }
      *reinterpret_cast<uint4*>(st + 16 * lane) = v;
    }
    __syncwarp();
    const uint2 lo = *reinterpret_cast<const uint2*>(st + cpos);
    const uint2 hi = j < 7 ? *reinterpret_cast<const uint2*>(st + cpos + 8) : make_uint2(0, 0);
    __syncwarp();  // the buffer is refilled on the next pass
    put_group(a.fifo_rs + ((s * n + r) * a.gps + gi) * kGroupLines, make_uint4(lo.x, lo.y, hi.x, hi.y), flag_rs);
  }
  pdl_trigger();

  // B: I own segment r: reduce each group over the ranks in rank order and
  // send it to every rank
  for (uint64_t gi = wid; alive && gi < a.gps; gi += wstride) {
    auto src = [&](int q) { return a.fifo_rs + ((static_cast<uint64_t>(r) * n + q) * a.gps + gi) * kGroupLines; };
    for (int q = 0; q < n && alive; ++q) alive = wait_group(src(q), flag_rs);
    if (!alive) break;
    acquire();  // one fence for all n sources
    A acc[VN];
    for (int q = 0; q < n; ++q) {
      Vec<DT> x;
      widen16<DT>(read_data(src(q)), x);
      if (q == 0) {
#pragma unroll
        for (int i = 0; i < VN; ++i) acc[i] = x.v[i];
      } else {
#pragma unroll
        for (int i = 0; i < VN; ++i) acc[i] = op_step<OP>(acc[i], x.v[i]);
      }
    }
    Vec<DT> w;
#pragma unroll
    for (int i = 0; i < VN; ++i) w.v[i] = acc[i];
    const uint4 o = narrow16<DT>(w);
    // every destination's data, one fence, then every destination's flags
    for (int q = 0; q < n; ++q) {
      char* p = a.fifo_ag + ((static_cast<uint64_t>(q) * n + r) * a.gps + gi) * kGroupLines + 128 * l + 16 * j;
      if (j < 7) t128_st16(p, o);
      else t128_st8(p, o.x, o.y);
    }
    __syncwarp();
    if (j == 7) {
      t128_fence();
      for (int q = 0; q < n; ++q)
        t128_st64(a.fifo_ag + ((static_cast<uint64_t>(q) * n + r) * a.gps + gi) * kGroupLines + 128 * l + 120, flag_ag);
    }
  }

  // C: the reduced groups of every owner into my output
  for (uint64_t it = wid; alive && it < items; it += wstride) {
    const uint64_t s = it / a.gps, gi = it - s * a.gps;
    const char* grp = a.fifo_ag + ((static_cast<uint64_t>(r) * n + s) * a.gps + gi) * kGroupLines;
    if (!wait_group(grp, flag_ag)) {
      alive = false;
      break;
    }
    acquire();
    const uint4 v = read_data(grp);
    *reinterpret_cast<uint2*>(st + cpos) = make_uint2(v.x, v.y);
    if (j < 7) *reinterpret_cast<uint2*>(st + cpos + 8) = make_uint2(v.z, v.w);
    __syncwarp();
    if (lane < 30) {
      const uint64_t valid = valid_b(s);
      const uint64_t o = gi * kGroupData + 16 * lane;
      char* dst = a.out[r] + s * seg_b + o;
      const uint4 x = *reinterpret_cast<const uint4*>(st + 16 * lane);
      if (o + 16 <= valid) {
        st16(dst, x);
      } else if (o < valid) {
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int i = 0; i < VN; ++i)
          if (o + (i + 1) * ES <= valid)
            *reinterpret_cast<S*>(dst + i * ES) = static_cast<S>(w[i * ES / 4] >> (8 * (i * ES % 4)));
      }
    }
    __syncwarp();
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

static uint64_t t128_gps(int n, size_t count, int es) {
  const size_t g = 16 / es;
  const size_t seg = ((count + n - 1) / n + g - 1) / g * g;
  return (seg * es + kGroupData - 1) / kGroupData;
}

size_t twoshot_ll128_workspace(int n, size_t count, int es) {
  return 256 + 2 * static_cast<size_t>(n) * n * t128_gps(n, count, es) * kGroupLines;
}

template <int DT, int OP>
static int launch_twoshot_ll128_t(TwoShotLL128Args& a, cudaStream_t s) {
  static int max_per_sm[COLL_MAX_RANKS] = {0};  // per device ordinal (benign race: same value)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= COLL_MAX_RANKS) dev = 0;
  if (max_per_sm[dev] == 0) {
    int v = 0;
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, k_twoshot_ll128<DT, OP>, kT128Threads, 0);
    if (e != cudaSuccess || v <= 0) {
      (void)cudaGetLastError();
      return launch_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
    }
    max_per_sm[dev] = v;
  }
  const int max_groups = max_per_sm[dev] * num_sms() / a.n;
  if (max_groups < 1) return COLL_ERR_UNSUPPORTED;  // more ranks than co-resident CTAs
  const uint64_t warps_needed = static_cast<uint64_t>(a.n) * a.gps;  // phase A and C items of one rank
  a.groups = static_cast<int>(std::min<uint64_t>((warps_needed + kT128Warps - 1) / kT128Warps, max_groups));
  if (a.groups < 1) a.groups = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(a.groups * a.n));
  cfg.blockDim = dim3(kT128Threads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_twoshot_ll128<DT, OP>, a);
  if (e != cudaSuccess) (void)cudaGetLastError();  // reported here; keep it from surfacing in a later call
  return launch_status(e);
}

template <int DT>
static int launch_twoshot_ll128_dt(TwoShotLL128Args& a, coll_op_t op, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_twoshot_ll128_t<DT, COLL_SUM>(a, s);
    case COLL_MAX: return launch_twoshot_ll128_t<DT, COLL_MAX>(a, s);
    case COLL_MIN: return launch_twoshot_ll128_t<DT, COLL_MIN>(a, s);
    case COLL_PROD: return launch_twoshot_ll128_t<DT, COLL_PROD>(a, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

int launch_twoshot_ll128(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt,
                         coll_op_t op, void* workspace, int* status, cudaStream_t s) {
  TwoShotLL128Args a{};
  for (int r = 0; r < n; ++r) {
    a.in[r] = in[r];
    a.out[r] = out[r];
  }
  const int es = elem_size(dt);
  const size_t g = 16 / es;
  a.seg = ((count + n - 1) / n + g - 1) / g * g;
  a.count = count;
  a.n = n;
  a.gps = t128_gps(n, count, es);
  a.status = status;
  a.hdr = static_cast<uint32_t*>(workspace);
  a.fifo_rs = static_cast<char*>(workspace) + 256;
  a.fifo_ag = a.fifo_rs + static_cast<size_t>(n) * n * a.gps * kGroupLines;
  switch (dt) {
    case COLL_BF16: return launch_twoshot_ll128_dt<COLL_BF16>(a, op, s);
    case COLL_FP16: return launch_twoshot_ll128_dt<COLL_FP16>(a, op, s);
    case COLL_FP32: return launch_twoshot_ll128_dt<COLL_FP32>(a, op, s);
    case COLL_INT32: return launch_twoshot_ll128_dt<COLL_INT32>(a, op, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

}  // namespace mvr
