// Element-wise reductions over virtual ranks: the owner-segment two-shot
// all-reduce, the one-shot all-reduce, reduce-scatter, reduce, and the
// reduce-scatter steps of the ring all-reduce.
//
// Per element: acc = widen(x_0); acc = acc (op) widen(x_r) for r = 1..N-1 in
// IEEE binary32 (no contraction: __fadd_rn / __fmul_rn); one rounding to the
// storage type.  Each thread owns 16 bytes of every rank (8 bf16 lanes) and
// issues its loads before combining them (all N for the rank counts compiled
// as such, eight at a time for any other), so up to 8 x 16 bytes per thread
// are in flight; outputs are plain 16-byte stores.
//
// Slices: blockIdx.x = part * nslices + slice.  For the two-shot all-reduce a
// slice is owner s's segment ("From NCCL Ring LL to PCIe IPC AllReduce",
// section "Pro5000 ?": owner s sums segment s over all ranks and sends it to
// every rank); for reduce-scatter it is output block r (vLLM collectives
// tutorial, section 5.1); for the one-shot all-reduce it is output rank q
// recomputing the whole range (interleaving the slices keeps the N readers of
// one tile close together in time, so the repeated reads hit L2).
#pragma once

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace mvr {

template <int MODE>
__device__ __forceinline__ char* out_ptr(const ReduceArgs& a, int q_or_slice, uint64_t byte,
                                         uint64_t lo_byte) {
  if constexpr (MODE == M_BLOCK) return a.out[q_or_slice] + (byte - lo_byte);
  else if constexpr (MODE == M_SAME) return a.out[0] + byte;
  else return a.out[q_or_slice] + byte;  // M_ALL (q) and M_ONESHOT (slice)
}

template <int DT, int OP, int MODE>
__device__ __forceinline__ void reduce_one(const ReduceArgs& a, int slice, uint64_t lo, uint64_t e,
                                           int n) {
  using S = typename Elem<DT>::S;
  constexpr int ES = Elem<DT>::kSize;
  const uint64_t byte = e * ES;
  auto acc = widen1<DT>(*reinterpret_cast<const S*>(a.in[0] + byte));
  for (int r = 1; r < n; ++r) acc = op_step<OP>(acc, widen1<DT>(*reinterpret_cast<const S*>(a.in[r] + byte)));
  const S o = narrow1<DT>(acc);
  if constexpr (MODE == M_ALL) {
    for (int q = 0; q < a.nout; ++q) *reinterpret_cast<S*>(out_ptr<MODE>(a, q, byte, lo * ES)) = o;
  } else {
    *reinterpret_cast<S*>(out_ptr<MODE>(a, slice, byte, lo * ES)) = o;
  }
}

template <int MODE>
__device__ __forceinline__ void slice_range(const ReduceArgs& a, int slice, uint64_t& lo, uint64_t& hi) {
  if constexpr (MODE == M_ONESHOT) {
    lo = 0;
    hi = a.count;
  } else {
    lo = static_cast<uint64_t>(slice) * a.seg;
    if (lo > a.count) lo = a.count;
    hi = lo + a.seg;
    if (hi > a.count) hi = a.count;
  }
}

template <int DT, int OP, int NR, int MODE>
__global__ void __launch_bounds__(kThreads) k_reduce_vec(const __grid_constant__ ReduceArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int VN = Vec<DT>::kN;
  constexpr int ES = Elem<DT>::kSize;
  const int n = NR > 0 ? NR : a.nin;
  const int slice = blockIdx.x % a.nslices;
  const int part = blockIdx.x / a.nslices;
  const int parts = gridDim.x / a.nslices;
  uint64_t lo, hi;
  slice_range<MODE>(a, slice, lo, hi);
  const uint64_t nv = (hi - lo) / VN;
  const uint64_t stride = static_cast<uint64_t>(parts) * blockDim.x;
  for (uint64_t v = static_cast<uint64_t>(part) * blockDim.x + threadIdx.x; v < nv; v += stride) {
    const uint64_t byte = (lo + v * VN) * ES;
    Vec<DT> acc;
    if constexpr (NR > 0) {
      uint4 x[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) x[r] = ld16(a.in[r] + byte);
      widen16<DT>(x[0], acc);
#pragma unroll
      for (int r = 1; r < NR; ++r) step16<DT, OP>(acc, x[r]);
    } else {
      // any rank count: loads issued eight at a time before they are
      // combined (in rank order), so a thread waits once per eight ranks
      constexpr int B = 8;
      for (int r0 = 0; r0 < n; r0 += B) {
        uint4 x[B];
#pragma unroll
        for (int i = 0; i < B; ++i)
          if (r0 + i < n) x[i] = ld16(a.in[r0 + i] + byte);
#pragma unroll
        for (int i = 0; i < B; ++i) {
          if (r0 + i >= n) break;
          if (r0 + i == 0) widen16<DT>(x[0], acc);
          else step16<DT, OP>(acc, x[i]);
        }
      }
    }
    const uint4 o = narrow16<DT>(acc);
    if constexpr (MODE == M_ALL) {
      const int nout = NR > 0 ? NR : a.nout;
#pragma unroll
      for (int q = 0; q < nout; ++q) st16(out_ptr<MODE>(a, q, byte, lo * ES), o);
    } else {
      st16(out_ptr<MODE>(a, slice, byte, lo * ES), o);
    }
  }
  if (part == 0) {  // ragged end of the slice: fewer than 16 bytes
    const uint64_t e = lo + nv * VN + threadIdx.x;
    if (e < hi) reduce_one<DT, OP, MODE>(a, slice, lo, e, n);
  }
}

template <int DT, int OP, int MODE>
__global__ void __launch_bounds__(kThreads) k_reduce_scalar(const __grid_constant__ ReduceArgs a) {
  pdl_wait();
  pdl_trigger();
  const int slice = blockIdx.x % a.nslices;
  const int part = blockIdx.x / a.nslices;
  const int parts = gridDim.x / a.nslices;
  uint64_t lo, hi;
  slice_range<MODE>(a, slice, lo, hi);
  const uint64_t stride = static_cast<uint64_t>(parts) * blockDim.x;
  for (uint64_t e = lo + static_cast<uint64_t>(part) * blockDim.x + threadIdx.x; e < hi; e += stride)
    reduce_one<DT, OP, MODE>(a, slice, lo, e, a.nin);
}

// ------------------------------------------------------------ ring steps ----
// Step k (1 .. N-1) of the reduce-scatter phase: chunk c, started on rank
// c+1, arrives at rank (c+1+k) mod N, which combines its own values with the
// partial that travelled in the arithmetic type; the last step rounds and
// writes the finished chunk to rank c's output.
template <int DT, int OP, bool VEC>
__global__ void __launch_bounds__(kThreads) k_ring_rs(const __grid_constant__ RingStepArgs a) {
  using A = typename Elem<DT>::A;
  using S = typename Elem<DT>::S;
  constexpr int VN = Vec<DT>::kN;
  constexpr int ES = Elem<DT>::kSize;
  const int c = blockIdx.x % a.n;
  const int part = blockIdx.x / a.n;
  const int parts = gridDim.x / a.n;
  uint64_t lo = static_cast<uint64_t>(c) * a.seg;
  if (lo > a.count) lo = a.count;
  uint64_t hi = lo + a.seg;
  if (hi > a.count) hi = a.count;
  const int r = (c + 1 + a.k) % a.n;
  const int r0 = (c + 1) % a.n;
  const bool first = a.k == 1;
  const bool last = a.k == a.n - 1;
  A* part_buf = reinterpret_cast<A*>(a.partial);
  const uint64_t stride = static_cast<uint64_t>(parts) * blockDim.x;
  const uint64_t v0 = static_cast<uint64_t>(part) * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  uint64_t scalar_from = lo;
  if constexpr (VEC) {
    const uint64_t nv = (hi - lo) / VN;
    for (uint64_t v = v0; v < nv; v += stride) {
      const uint64_t e = lo + v * VN;
      Vec<DT> acc;
      if (first) {
        widen16<DT>(ld16(a.in[r0] + e * ES), acc);
      } else {
        const uint4* pp = reinterpret_cast<const uint4*>(part_buf + e);
#pragma unroll
        for (int j = 0; j < VN / 4; ++j) {
          const uint4 w = pp[j];
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if constexpr (std::is_same<A, float>::value) acc.v[4 * j + i] = __uint_as_float(ww[i]);
            else acc.v[4 * j + i] = static_cast<int32_t>(ww[i]);
          }
        }
      }
      step16<DT, OP>(acc, ld16(a.in[r] + e * ES));
      if (last) {
        st16(a.out[c] + e * ES, narrow16<DT>(acc));
      } else {
        uint4* pp = reinterpret_cast<uint4*>(part_buf + e);
#pragma unroll
        for (int j = 0; j < VN / 4; ++j) {
          uint32_t ww[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if constexpr (std::is_same<A, float>::value) ww[i] = __float_as_uint(acc.v[4 * j + i]);
            else ww[i] = static_cast<uint32_t>(acc.v[4 * j + i]);
          }
          pp[j] = make_uint4(ww[0], ww[1], ww[2], ww[3]);
        }
      }
    }
    scalar_from = lo + nv * VN;
    if (part != 0) return;
  }
  const uint64_t s0 = VEC ? scalar_from + threadIdx.x : lo + static_cast<uint64_t>(part) * blockDim.x + threadIdx.x;
  const uint64_t sstride = VEC ? static_cast<uint64_t>(blockDim.x) : stride;
  for (uint64_t e = s0; e < hi; e += sstride) {
    A acc = first ? widen1<DT>(*reinterpret_cast<const S*>(a.in[r0] + e * ES)) : part_buf[e];
    acc = op_step<OP>(acc, widen1<DT>(*reinterpret_cast<const S*>(a.in[r] + e * ES)));
    if (last) *reinterpret_cast<S*>(a.out[c] + e * ES) = narrow1<DT>(acc);
    else part_buf[e] = acc;
  }
}

// ------------------------------------------------------------- launchers ----

template <int DT, int OP, int NR>
int launch_reduce_nr(const ReduceArgs& a, int mode, bool vec, int bps, cudaStream_t s) {
  void (*fn)(ReduceArgs) = nullptr;
  if (vec) {
    switch (mode) {
      case M_ALL: fn = k_reduce_vec<DT, OP, NR, M_ALL>; break;
      case M_BLOCK: fn = k_reduce_vec<DT, OP, NR, M_BLOCK>; break;
      case M_SAME: fn = k_reduce_vec<DT, OP, NR, M_SAME>; break;
      default: fn = k_reduce_vec<DT, OP, NR, M_ONESHOT>; break;
    }
  } else {
    switch (mode) {
      case M_ALL: fn = k_reduce_scalar<DT, OP, M_ALL>; break;
      case M_BLOCK: fn = k_reduce_scalar<DT, OP, M_BLOCK>; break;
      case M_SAME: fn = k_reduce_scalar<DT, OP, M_SAME>; break;
      default: fn = k_reduce_scalar<DT, OP, M_ONESHOT>; break;
    }
  }
  // one vector per thread (blocks_per_slice), the slices interleaved; the
  // one-shot keeps a resident grid, so that the N readers of a tile run
  // together and L2 serves the repeats (a full grid measured 17.4 -> 20.1 us
  // at 8 x 3.5 MiB)
  if (mode == M_ONESHOT) {
    const int res = resident_ctas(reinterpret_cast<const void*>(fn), kThreads, 0);
    if (static_cast<int64_t>(a.nslices) * bps > res) bps = std::max(1, res / a.nslices);
  }
  launch_pdl(fn, dim3(static_cast<unsigned>(a.nslices * bps)), dim3(kThreads), 0, s, a);
  return launch_status(cudaGetLastError());
}

template <int DT, int OP>
int launch_reduce_op(const ReduceArgs& a, int mode, bool vec, int bps, cudaStream_t s) {
  if (vec && OP == COLL_SUM) {
    if (a.nin == 2) return launch_reduce_nr<DT, OP, 2>(a, mode, vec, bps, s);
    if (a.nin == 4) return launch_reduce_nr<DT, OP, 4>(a, mode, vec, bps, s);
    if (a.nin == 8) return launch_reduce_nr<DT, OP, 8>(a, mode, vec, bps, s);
  }
  return launch_reduce_nr<DT, OP, 0>(a, mode, vec, bps, s);
}

template <int DT>
int launch_reduce_dt(const ReduceArgs& a, coll_op_t op, int mode, bool vec, int bps, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_reduce_op<DT, COLL_SUM>(a, mode, vec, bps, s);
    case COLL_MAX: return launch_reduce_op<DT, COLL_MAX>(a, mode, vec, bps, s);
    case COLL_MIN: return launch_reduce_op<DT, COLL_MIN>(a, mode, vec, bps, s);
    case COLL_PROD: return launch_reduce_op<DT, COLL_PROD>(a, mode, vec, bps, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

template <int DT, int OP>
int launch_ring_op(const RingStepArgs& a, bool vec, cudaStream_t s) {
  const uint64_t per = a.seg / (vec ? Vec<DT>::kN : 1);
  uint64_t want = (per + kThreads - 1) / kThreads;
  const uint64_t cap = static_cast<uint64_t>(num_sms()) * 8 / a.n;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  const dim3 grid(static_cast<unsigned>(a.n * want));
  if (vec) launch_pdl(k_ring_rs<DT, OP, true>, dim3(grid), dim3(kThreads), 0, s, a);
  else launch_pdl(k_ring_rs<DT, OP, false>, dim3(grid), dim3(kThreads), 0, s, a);
  return launch_status(cudaGetLastError());
}

template <int DT>
int launch_ring_dt(const RingStepArgs& a, coll_op_t op, bool vec, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_ring_op<DT, COLL_SUM>(a, vec, s);
    case COLL_MAX: return launch_ring_op<DT, COLL_MAX>(a, vec, s);
    case COLL_MIN: return launch_ring_op<DT, COLL_MIN>(a, vec, s);
    case COLL_PROD: return launch_ring_op<DT, COLL_PROD>(a, vec, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

}  // namespace mvr

#define MVR_REDUCE_INSTANCE(NAME, DT)                                                         \
  namespace mvr {                                                                             \
  int launch_reduce_##NAME(const ReduceArgs& a, coll_op_t op, int mode, bool vec, int bps,    \
                           cudaStream_t s) {                                                  \
    return launch_reduce_dt<DT>(a, op, mode, vec, bps, s);                                    \
  }                                                                                           \
  int launch_ring_##NAME(const RingStepArgs& a, coll_op_t op, bool vec, cudaStream_t s) {     \
    return launch_ring_dt<DT>(a, op, vec, s);                                                 \
  }                                                                                           \
  }
