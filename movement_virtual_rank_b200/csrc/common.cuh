// Shared device-side helpers of the virtual-rank collectives (sm_100a).
//
// Element types, exact widening to the arithmetic type, the single rounding
// back to storage, the per-step reduction operators, 16-byte memory access
// and device-status reporting.  Every kernel file includes this header;
// nothing here is shared with the CPU oracle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "coll.h"
#include "internal.h"

namespace mvr {

constexpr int kMaxRanks = COLL_MAX_RANKS;
constexpr int kThreads = kBlockThreads;

enum ReduceMode : int {
  M_ALL = 0,      // owner-segment two-shot: write every output rank at the same offset
  M_BLOCK = 1,    // reduce-scatter: slice y goes to out[y] at the offset within the slice
  M_SAME = 2,     // reduce to one rank: out[0] at the same offset
  M_ONESHOT = 3,  // slice y = output rank y, each recomputing the whole range
};

// ---------------------------------------------------------------- types ----

template <int DT>
struct Elem;

template <>
struct Elem<COLL_BF16> {
  using S = uint16_t;  // storage bits
  using A = float;     // arithmetic type
  static constexpr int kSize = 2;
};
template <>
struct Elem<COLL_FP16> {
  using S = uint16_t;
  using A = float;
  static constexpr int kSize = 2;
};
template <>
struct Elem<COLL_FP32> {
  using S = uint32_t;
  using A = float;
  static constexpr int kSize = 4;
};
template <>
struct Elem<COLL_INT32> {
  using S = uint32_t;
  using A = int32_t;
  static constexpr int kSize = 4;
};

// exact widening of one storage element
template <int DT>
__device__ __forceinline__ typename Elem<DT>::A widen1(typename Elem<DT>::S s) {
  if constexpr (DT == COLL_BF16) {
    return __uint_as_float(static_cast<uint32_t>(s) << 16);
  } else if constexpr (DT == COLL_FP16) {
    return __half2float(__ushort_as_half(s));
  } else if constexpr (DT == COLL_FP32) {
    return __uint_as_float(s);
  } else {
    return static_cast<int32_t>(s);
  }
}

// the one rounding: round to nearest even (hardware cvt.rn), NaN -> canonical
template <int DT>
__device__ __forceinline__ typename Elem<DT>::S narrow1(typename Elem<DT>::A a) {
  if constexpr (DT == COLL_BF16) {
    if (a != a) return 0x7FC0;
    return __bfloat16_as_ushort(__float2bfloat16_rn(a));
  } else if constexpr (DT == COLL_FP16) {
    if (a != a) return 0x7E00;
    return __half_as_ushort(__float2half_rn(a));
  } else if constexpr (DT == COLL_FP32) {
    return a != a ? 0x7FC00000u : __float_as_uint(a);
  } else {
    return static_cast<uint32_t>(a);
  }
}

// two elements packed in one 32-bit word (16-bit types)
__device__ __forceinline__ uint32_t narrow2_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  if (lo != lo) r = (r & 0xFFFF0000u) | 0x00007FC0u;
  if (hi != hi) r = (r & 0x0000FFFFu) | 0x7FC00000u;
  return r;
}
__device__ __forceinline__ uint32_t narrow2_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  if (lo != lo) r = (r & 0xFFFF0000u) | 0x00007E00u;
  if (hi != hi) r = (r & 0x0000FFFFu) | 0x7E000000u;
  return r;
}

// ---------------------------------------------------------- operators ----

template <int OP, typename A>
__device__ __forceinline__ A op_step(A acc, A v) {
  if constexpr (std::is_same<A, float>::value) {
    if constexpr (OP == COLL_SUM) return __fadd_rn(acc, v);
    if constexpr (OP == COLL_PROD) return __fmul_rn(acc, v);
    if constexpr (OP == COLL_MAX) return (!(acc != acc) && ((v != v) || (v > acc))) ? v : acc;
    if constexpr (OP == COLL_MIN) return (!(acc != acc) && ((v != v) || (v < acc))) ? v : acc;
  } else {
    if constexpr (OP == COLL_SUM)
      return static_cast<int32_t>(static_cast<uint32_t>(acc) + static_cast<uint32_t>(v));
    if constexpr (OP == COLL_PROD)
      return static_cast<int32_t>(static_cast<uint32_t>(acc) * static_cast<uint32_t>(v));
    if constexpr (OP == COLL_MAX) return v > acc ? v : acc;
    if constexpr (OP == COLL_MIN) return v < acc ? v : acc;
  }
}

// ---------------------------------------------- 16-byte vectors of elements

template <int DT>
struct Vec {
  static constexpr int kN = 16 / Elem<DT>::kSize;  // elements per 16 bytes
  using A = typename Elem<DT>::A;
  A v[kN];
};

template <int DT>
__device__ __forceinline__ void widen16(const uint4& x, Vec<DT>& o) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  if constexpr (DT == COLL_BF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o.v[2 * i] = __uint_as_float(w[i] << 16);
      o.v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else if constexpr (DT == COLL_FP16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o.v[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xFFFFu)));
      o.v[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
    }
  } else if constexpr (DT == COLL_FP32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) o.v[i] = __uint_as_float(w[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) o.v[i] = static_cast<int32_t>(w[i]);
  }
}

template <int DT>
__device__ __forceinline__ uint4 narrow16(const Vec<DT>& a) {
  uint32_t w[4];
  if constexpr (DT == COLL_BF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = narrow2_bf16(a.v[2 * i], a.v[2 * i + 1]);
  } else if constexpr (DT == COLL_FP16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = narrow2_f16(a.v[2 * i], a.v[2 * i + 1]);
  } else if constexpr (DT == COLL_FP32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = a.v[i] != a.v[i] ? 0x7FC00000u : __float_as_uint(a.v[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = static_cast<uint32_t>(a.v[i]);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int DT, int OP>
__device__ __forceinline__ void step16(Vec<DT>& acc, const uint4& x) {
  Vec<DT> v;
  widen16<DT>(x, v);
#pragma unroll
  for (int i = 0; i < Vec<DT>::kN; ++i) acc.v[i] = op_step<OP>(acc.v[i], v.v[i]);
}

// ------------------------------------------------------ memory access ----

// read-only streaming load (the inputs are never written by the same kernel
// at an address another thread reads)
__device__ __forceinline__ uint4 ld16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void st16(void* p, const uint4& v) {
  *reinterpret_cast<uint4*>(p) = v;
}
__device__ __forceinline__ uint2 ld8(const void* p) {
  return __ldg(reinterpret_cast<const uint2*>(p));
}
__device__ __forceinline__ void st8(void* p, const uint2& v) {
  *reinterpret_cast<uint2*>(p) = v;
}

template <int U>
struct UnitT;
template <>
struct UnitT<16> { using T = uint4; };
template <>
struct UnitT<8> { using T = uint2; };
template <>
struct UnitT<4> { using T = uint32_t; };
template <>
struct UnitT<2> { using T = uint16_t; };
template <>
struct UnitT<1> { using T = uint8_t; };

template <int U>
__device__ __forceinline__ typename UnitT<U>::T ldu(const char* p) {
  if constexpr (U == 16) return __ldg(reinterpret_cast<const uint4*>(p));
  else if constexpr (U == 8) return __ldg(reinterpret_cast<const uint2*>(p));
  else if constexpr (U == 4) return __ldg(reinterpret_cast<const unsigned int*>(p));
  else if constexpr (U == 2) return __ldg(reinterpret_cast<const unsigned short*>(p));
  else return static_cast<uint8_t>(__ldg(reinterpret_cast<const unsigned char*>(p)));
}
template <int U>
__device__ __forceinline__ void stu(char* p, const typename UnitT<U>::T& v) {
  *reinterpret_cast<typename UnitT<U>::T*>(p) = v;
}

// ------------------------------------------- programmatic dependent launch ----
// Every kernel is launched with programmatic stream serialisation allowed, so
// the hardware may schedule its CTAs while the previous kernel in the stream
// is still draining.  pdl_wait() (griddepcontrol.wait) blocks until that
// predecessor has completed and its memory is visible, and is the first thing
// every kernel does; it returns at once when there is no such predecessor.
// pdl_trigger() lets the next kernel in the stream start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------ device status ----

__device__ __forceinline__ void report(int* status, int code, int count) {
  if (status == nullptr || count == 0) return;
  atomicCAS(status, 0, code);
  atomicAdd(status + 1, count);
}

// warp-aggregated report: every lane passes its own count
__device__ __forceinline__ void report_warp(int* status, int code, int count) {
  if (status == nullptr) return;
  const unsigned any = __ballot_sync(0xFFFFFFFFu, count != 0);
  if (any == 0) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) count += __shfl_xor_sync(0xFFFFFFFFu, count, o);
  if ((threadIdx.x & 31) == 0) report(status, code, count);
}

}  // namespace mvr
