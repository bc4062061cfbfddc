// The ragged end of a ring all-reduce, shared by the one-launch ring forms
// whose hops move whole 16-byte vectors only (RING_CTA, RING_LANE).
#pragma once

#include "common.cuh"

namespace mvr {

// The elements after the message's last whole vector (fewer than VN, all in
// chunk ct): one thread each adds them in that chunk's ring order (ranks
// ct+1, ..., n-1, 0, ..., ct) with the same partial type and the one rounding
// at the end (WIRE: rounding to the storage type after every addition, as
// each hop of RING_WIRE does), and stores the result to every rank.  Each
// element is touched by its own thread only, so in place is safe.
template <int DT, int OP, bool WIRE = false, typename Args>
__device__ void ring_tail(const Args& a, int lane) {
  using S = typename Elem<DT>::S;
  constexpr int VN = Vec<DT>::kN;
  constexpr int ES = Elem<DT>::kSize;
  const uint64_t vcount = a.count / VN * VN;
  const uint64_t e = vcount + static_cast<uint64_t>(lane);
  if (e >= a.count) return;
  const int n = a.n;
  const int ct = static_cast<int>(vcount / a.seg);
  int q = ct + 1 == n ? 0 : ct + 1;
  auto acc = widen1<DT>(*reinterpret_cast<const S*>(a.in[q] + e * ES));
  for (int j = 1; j < n; ++j) {
    q = q + 1 == n ? 0 : q + 1;
    acc = op_step<OP>(acc, widen1<DT>(*reinterpret_cast<const S*>(a.in[q] + e * ES)));
    if constexpr (WIRE) acc = widen1<DT>(narrow1<DT>(acc));
  }
  const S o = narrow1<DT>(acc);
  for (int r = 0; r < n; ++r) *reinterpret_cast<S*>(a.out[r] + e * ES) = o;
}

}  // namespace mvr
