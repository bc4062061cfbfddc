// Ring all-reduce with the virtual ranks as thread groups of one CTA: the hop
// from rank r to rank r+1 is a store into shared memory of the same SM and an
// arrive on an mbarrier there, the shortest hand-off the GPU has.
//
// The schedule, chunk order, fp32 partials and the single rounding are those
// of coll_all_reduce(RING) (TP communication essay; NCCL's ring kernel named
// in "From NCCL Ring LL to PCIe IPC AllReduce"), so the result is
// bit-identical.  A CTA holds all N ranks, TW threads each (thread t of
// group r plays rank r for VN elements of every chunk of a tile of TW x VN
// elements); the CTAs of the grid walk the tiles with a stride.
//
// Hop transport.  For each of the 2N-2 hops of a tile, sender thread t
// stores its values into slot h mod N of the receiving group (fp32 partials
// in the reduce-scatter hops, laid out piece-major so that a warp's 16-byte
// stores are contiguous; the rounded storage-type values in the all-gather
// hops) and arrives, with release semantics at CTA scope, on that slot's
// mbarrier, which completes a phase after TW arrivals and re-arms itself;
// the receiving threads wait on it (acquire).  Hops are numbered without a
// break from tile to tile and, as in the cluster form, the ring's own
// dependencies keep a sender within N-1 hops of its receiver, so N slots per
// group need no credits.
//
// The kernel is bound by instruction issue, not by HBM, so the tiles that are
// full in every chunk (those that end within the last chunk, the shortest)
// take a path with no bounds checks and with chunk offsets stepped by one
// addition; the other tiles check each vector against its chunk's end.
//
// Every wait is bounded: a thread whose wait runs out raises COLL_DEV_TIMEOUT
// and sets the CTA's abort word; the others stop at their next wait, and all
// meet at the final barrier.  Nothing leaves the SM but the loads of inputs
// and the stores of outputs.
#include <algorithm>

#include "bulk.cuh"
#include "common.cuh"
#include "internal.h"

namespace mvr {

constexpr int kRtMaxRanks = 8;
constexpr long long kRtBudgetCycles = 1ll << 28;  // about 0.14 s per wait

struct RingCtaArgs {
  const char* in[kMaxRanks];
  char* out[kMaxRanks];
  uint64_t count, seg, tiles;
  uint64_t full_tiles;  // tiles [0, full_tiles) are full in every chunk
  int n;
  int* status;
};

__device__ __forceinline__ void rt_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool rt_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

template <int DT, int OP, int TW>
__global__ void __launch_bounds__(TW * kRtMaxRanks) k_ring_cta(const __grid_constant__ RingCtaArgs a) {
  using A = typename Elem<DT>::A;
  using S = typename Elem<DT>::S;
  constexpr int VN = Vec<DT>::kN;  // elements per thread (16 bytes of input)
  constexpr int NQ = VN / 4;       // 16-byte pieces of fp32 / int32 partials per thread
  constexpr int ES = Elem<DT>::kSize;
  constexpr uint64_t TE = static_cast<uint64_t>(TW) * VN;  // elements of a chunk per tile
  constexpr uint32_t kSlotU4 = TW * NQ;                    // slot size in 16-byte units
  extern __shared__ __align__(16) uint4 slot_buf[];        // [receiving group][slot][kSlotU4]
  __shared__ __align__(8) uint64_t bar[kRtMaxRanks * kRtMaxRanks];  // [receiving group][slot]
  __shared__ uint32_t abort_word;
  const int n = a.n;
  const int r = threadIdx.x / TW;
  const int t = threadIdx.x % TW;
  if (threadIdx.x == 0) {
    abort_word = 0;
    for (int i = 0; i < n * n; ++i) mbar_init(&bar[i], TW);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  const int nxt = (r + 1) % n;
  uint4* const my_slots = slot_buf + static_cast<size_t>(r) * n * kSlotU4;
  uint4* const next_slots = slot_buf + static_cast<size_t>(nxt) * n * kSlotU4;
  uint64_t* const my_bar = bar + r * n;
  uint64_t* const next_bar = bar + nxt * n;
  bool alive = true;

  // chunk c of a rank starts c * seg elements in; step k of the
  // reduce-scatter handles chunk (r - 1 - k) mod n, all-gather hop j chunk
  // (r - j) mod n: both walk the chunks downwards, wrapping from 0 to n - 1
  const int64_t seg_b = static_cast<int64_t>(a.seg) * ES;
  const int64_t top_b = static_cast<int64_t>(n - 1) * seg_b;
  const int c0 = r == 0 ? n - 1 : r - 1;
  const int64_t off0 = static_cast<int64_t>(c0) * seg_b;
  const int64_t off_r = static_cast<int64_t>(r) * seg_b;
  auto down = [&](int64_t off) { return off == 0 ? top_b : off - seg_b; };
  const char* const in_r = a.in[r];
  char* const out_r = a.out[r];
  auto chunk_end = [&](int c) { return min(static_cast<uint64_t>(c) * a.seg + a.seg, a.count); };

  auto to_bits = [](A x) -> uint32_t {
    if constexpr (std::is_same<A, float>::value) return __float_as_uint(x);
    else return static_cast<uint32_t>(x);
  };
  auto from_bits = [](uint32_t u) -> A {
    if constexpr (std::is_same<A, float>::value) return __uint_as_float(u);
    else return static_cast<A>(static_cast<int32_t>(u));
  };

  uint32_t js = 0;          // slot of the next hop to send
  uint32_t jr = 0, pr = 0;  // slot and phase parity of the next hop to receive
  auto send_wide = [&](const A (&v)[VN]) {
    uint4* d = next_slots + js * kSlotU4 + t;
#pragma unroll
    for (int q = 0; q < NQ; ++q)
      d[q * TW] = make_uint4(to_bits(v[4 * q]), to_bits(v[4 * q + 1]), to_bits(v[4 * q + 2]), to_bits(v[4 * q + 3]));
    rt_arrive(&next_bar[js]);
    js = js + 1 == static_cast<uint32_t>(n) ? 0 : js + 1;
  };
  auto send_narrow = [&](const uint4& w) {
    next_slots[js * kSlotU4 + t] = w;
    rt_arrive(&next_bar[js]);
    js = js + 1 == static_cast<uint32_t>(n) ? 0 : js + 1;
  };
  auto wait_next = [&]() -> bool {
    if (!rt_try_wait(&my_bar[jr], pr)) {
      const long long t0 = clock64();
      while (!rt_try_wait(&my_bar[jr], pr)) {
        if (*reinterpret_cast<volatile uint32_t*>(&abort_word) != 0) return false;
        if (clock64() - t0 > kRtBudgetCycles) {
          report(a.status, COLL_DEV_TIMEOUT, 1);
          *reinterpret_cast<volatile uint32_t*>(&abort_word) = 1;
          return false;
        }
      }
    }
    return true;
  };
  auto advance = [&]() {
    if (++jr == static_cast<uint32_t>(n)) {
      jr = 0;
      pr ^= 1;
    }
  };
  auto recv_wide = [&](A (&v)[VN]) -> bool {
    if (!wait_next()) return false;
    const uint4* p = my_slots + jr * kSlotU4 + t;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const uint4 x = p[q * TW];
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
    w = my_slots[jr * kSlotU4 + t];
    advance();
    return true;
  };
  // this thread's inputs of a tile, in reduce-scatter step order
  auto fetch = [&](uint64_t tile, uint4 (&dst)[kRtMaxRanks]) {
    const uint64_t e = tile * TE + static_cast<uint64_t>(t) * VN;
    const char* base = in_r + e * ES;
    int64_t off = off0;
    int c = c0;
    const bool full = tile < a.full_tiles;
#pragma unroll
    for (int k = 0; k < kRtMaxRanks; ++k) {
      dst[k] = make_uint4(0, 0, 0, 0);
      if (k < n) {
        if (full || static_cast<uint64_t>(c) * a.seg + e + VN <= chunk_end(c)) dst[k] = ld16(base + off);
        off = down(off);
        c = c == 0 ? n - 1 : c - 1;
      }
    }
  };

  // A slot is refilled only after its previous hop was read (the argument of
  // the cluster form: the sender's hop h depends, thread by thread, on this
  // group's hop h - n + 1, sent only after reading hop h - n); and a phase
  // cannot take an arrival of the hop n later before all TW arrivals of its
  // own hop, for the same reason.
  const uint64_t G = gridDim.x;
  uint4 pre[kRtMaxRanks];
  fetch(blockIdx.x, pre);
  for (uint64_t tile = blockIdx.x; tile < a.tiles && alive; tile += G) {
    const uint64_t e = tile * TE + static_cast<uint64_t>(t) * VN;
    const bool full = tile < a.full_tiles;
    uint4 nx[kRtMaxRanks];
    if (tile + G < a.tiles) fetch(tile + G, nx);
    else
#pragma unroll
      for (int k = 0; k < kRtMaxRanks; ++k) nx[k] = make_uint4(0, 0, 0, 0);
    const char* const in_e = in_r + e * ES;
    char* const out_e = out_r + e * ES;

    // my values for reduce-scatter step k, chunk c (prefetched vector, or
    // the ragged tail of a chunk element by element)
    auto mine = [&](int k, int c, A (&v)[VN]) {
      const uint64_t gi = static_cast<uint64_t>(c) * a.seg + e;
      const uint64_t end = chunk_end(c);
      if (full || gi + VN <= end) {
        Vec<DT> w;
        widen16<DT>(pre[k], w);
#pragma unroll
        for (int i = 0; i < VN; ++i) v[i] = w.v[i];
      } else {
#pragma unroll
        for (int i = 0; i < VN; ++i)
          v[i] = gi + i < end ? widen1<DT>(*reinterpret_cast<const S*>(in_e + (gi - e + i) * ES)) : A(0);
      }
    };
    // store a rounded 16-byte vector of chunk c at byte offset off (= c * seg_b)
    auto put = [&](int c, int64_t off, const uint4& w) {
      if (full) {
        st16(out_e + off, w);
        return;
      }
      const uint64_t gi = static_cast<uint64_t>(c) * a.seg + e;
      const uint64_t end = chunk_end(c);
      if (gi + VN <= end) {
        st16(out_e + off, w);
      } else {
        const S* sv = reinterpret_cast<const S*>(&w);
#pragma unroll
        for (int i = 0; i < VN; ++i)
          if (gi + i < end) *reinterpret_cast<S*>(out_e + off + i * ES) = sv[i];
      }
    };

    A p[VN];
    int c = c0;
    mine(0, c, p);
    send_wide(p);
#pragma unroll
    for (int k = 1; k < kRtMaxRanks; ++k) {
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
        put(r, off_r, fin);
        send_narrow(fin);
      }
    }
    int cj = r;
    int64_t offj = off_r;
    for (int j = 1; j < n && alive; ++j) {  // all-gather hops: chunk r - j arrives, is stored and passed on
      uint4 w;
      if (!recv_narrow(w)) {
        alive = false;
        break;
      }
      cj = cj == 0 ? n - 1 : cj - 1;
      offj = down(offj);
      put(cj, offj, w);
      if (j < n - 1) send_narrow(w);
    }
#pragma unroll
    for (int k = 0; k < kRtMaxRanks; ++k) pre[k] = nx[k];
  }
  __syncthreads();  // every store into this CTA's shared memory has landed before it leaves
}

template <int DT, int OP, int TW>
static int launch_ring_cta_t(RingCtaArgs a, cudaStream_t s) {
  constexpr int VN = Vec<DT>::kN;
  const uint64_t per_tile = static_cast<uint64_t>(TW) * VN;
  a.tiles = std::max<uint64_t>(1, (a.seg + per_tile - 1) / per_tile);
  // the last chunk is the shortest (possibly empty): a tile is full in every
  // chunk when it is full in that one
  const uint64_t lead = static_cast<uint64_t>(a.n - 1) * a.seg;
  a.full_tiles = a.count > lead ? (a.count - lead) / per_tile : 0;
  const size_t smem = static_cast<size_t>(a.n) * a.n * TW * VN * 4;
  static int smem_set[COLL_MAX_RANKS] = {0};  // per device ordinal: largest limit set so far
  const int st = allow_dynamic_smem(reinterpret_cast<const void*>(k_ring_cta<DT, OP, TW>), smem, smem_set);
  if (st != COLL_OK) return st;
  const uint64_t grid = std::min<uint64_t>(a.tiles, static_cast<uint64_t>(num_sms()) * 2);
  launch_pdl(k_ring_cta<DT, OP, TW>, dim3(static_cast<unsigned>(grid)), dim3(TW * a.n), smem, s, a);
  return launch_status(cudaGetLastError());
}

template <int DT>
static int launch_ring_cta_dt(const RingCtaArgs& a, coll_op_t op, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_ring_cta_t<DT, COLL_SUM, 32>(a, s);
    case COLL_MAX: return launch_ring_cta_t<DT, COLL_MAX, 32>(a, s);
    case COLL_MIN: return launch_ring_cta_t<DT, COLL_MIN, 32>(a, s);
    case COLL_PROD: return launch_ring_cta_t<DT, COLL_PROD, 32>(a, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

bool ring_cta_supported(int n) { return n >= 2 && n <= kRtMaxRanks; }

int launch_ring_cta(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                    int* status, cudaStream_t s) {
  RingCtaArgs a{};
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
    case COLL_BF16: return launch_ring_cta_dt<COLL_BF16>(a, op, s);
    case COLL_FP16: return launch_ring_cta_dt<COLL_FP16>(a, op, s);
    case COLL_FP32: return launch_ring_cta_dt<COLL_FP32>(a, op, s);
    case COLL_INT32: return launch_ring_cta_dt<COLL_INT32>(a, op, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

}  // namespace mvr
