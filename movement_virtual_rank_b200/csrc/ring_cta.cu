// Ring all-reduce with the virtual ranks as warps of one CTA: the hop from
// rank r to rank r+1 is a store into a shared-memory slot of the same SM,
// and every hop of the ring is one CTA-wide barrier.
//
// The schedule, chunk order, fp32 partials and the single rounding are those
// of coll_all_reduce(RING) (TP communication essay; NCCL's ring kernel named
// in "From NCCL Ring LL to PCIe IPC AllReduce"), so the result is
// bit-identical.  A CTA holds all N ranks, one warp each (lane t of warp r
// plays rank r for one 16-byte vector of every chunk of a tile of 32 vectors
// per chunk); each CTA of the grid takes one tile.
//
// Hops.  The ring of one tile is 2N-2 hops: N-1 reduce-scatter hops that
// carry the fp32 / int32 partials (laid out piece-major, so that each
// 16-byte store of a warp is contiguous), then N-1 all-gather hops that carry
// the rounded storage-type values.  At hop h every warp stores what it sends
// into the slot of the next warp in buffer h mod 2, the CTA passes one
// barrier, and every warp reads its own slot.  All ranks of a tile advance
// together, as the synchronous ring does; the barrier makes the stores of hop
// h visible to their readers, and the reads of hop h happen before the
// barrier of hop h+1, which every store of hop h+2 into the same buffer
// follows.  There is no spin-wait: a CTA-wide barrier cannot time out, and
// the kernel waits on nothing outside its own CTA.
//
// Inputs are staged in shared memory: each thread copies the vector of every
// reduce-scatter step of its tile into its own 16-byte cell with cp.async,
// all N copies in flight at once, and a CTA that walks a further tile
// refills cell k with that tile's step k as soon as step k has read it.  The
// grid has one CTA per tile, launched in order (a CTA walks further tiles
// only beyond 2^30 of them): measured faster than a resident grid walking
// the tiles, with the next tile's inputs in the cells or in registers.
// Chunk boundaries are whole vectors, so every vector the hops carry lies
// wholly inside its chunk or wholly outside it -- except the one that holds
// the message's last count mod VN elements.  Those few elements (at most 7)
// are left out of the hops and reduced at the end by one warp in that
// chunk's ring order with the same fp32 partials, which gives the same bits.
// So the hot code moves only 16-byte vectors: tiles full in every chunk take
// it with no checks, the others with one predicate per vector.  Keeping
// element-wise code out of the per-step path matters: the steps are unrolled,
// and inlined element loops made the loop miss in the instruction cache.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "ring_tail.cuh"

namespace mvr {

constexpr int kRtMaxRanks = 8;

struct RingCtaArgs {
  const char* in[kMaxRanks];
  char* out[kMaxRanks];
  uint64_t count, seg, tiles;
  uint64_t full_tiles;  // tiles [0, full_tiles) are full in every chunk
  int n;
};

template <int DT>
__device__ __forceinline__ uint32_t a_to_bits(typename Elem<DT>::A x) {
  if constexpr (std::is_same<typename Elem<DT>::A, float>::value) return __float_as_uint(x);
  else return static_cast<uint32_t>(x);
}
template <int DT>
__device__ __forceinline__ typename Elem<DT>::A a_from_bits(uint32_t w) {
  if constexpr (std::is_same<typename Elem<DT>::A, float>::value) return __uint_as_float(w);
  else return static_cast<typename Elem<DT>::A>(static_cast<int32_t>(w));
}

// cp.async of one 16-byte vector into shared memory: `bytes` (16 or 0) read
// from src, the rest zero-filled; src must be a valid address either way
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int PENDING>
__device__ __forceinline__ void cp_async_wait_n() {
  asm volatile("cp.async.wait_group %0;" ::"n"(PENDING) : "memory");
}

// NR: the rank count at compile time (its loops unrolled and its waits
// immediate), or 0 for any count in 2..8.  WIRE: the reduce-scatter hops carry
// the partial rounded to the storage type (RING_WIRE) instead of fp32 /
// int32 (RING): each receiver widens it, adds its own values and rounds
// again before passing it on.
template <int DT, int OP, int MINB, typename OFF, int NR, bool WIRE>
__global__ void __launch_bounds__(kRtMaxRanks * 32, MINB) k_ring_cta(const __grid_constant__ RingCtaArgs a) {
  using A = typename Elem<DT>::A;
  constexpr int VN = Vec<DT>::kN;  // elements per 16-byte vector
  constexpr int NQ = WIRE ? 1 : VN / 4;  // 16-byte pieces a reduce-scatter hop carries per lane
  constexpr int ES = Elem<DT>::kSize;
  constexpr uint64_t TE = 32ull * VN;    // elements of one chunk per tile
  constexpr uint32_t kSlotU4 = 32 * NQ;  // one warp's hop slot, in 16-byte units
  constexpr int KMAX = NR > 0 ? NR : kRtMaxRanks;
  // [2 buffers][N receiving warps][kSlotU4] hop slots, then [N steps][32 N threads] own inputs
  extern __shared__ __align__(16) uint4 hop_buf[];
  const int n = NR > 0 ? NR : a.n;
  const int r = static_cast<int>(threadIdx.x >> 5);
  const int t = static_cast<int>(threadIdx.x & 31);
  pdl_wait();
  pdl_trigger();

  const int nxt = r + 1 == n ? 0 : r + 1;
  const uint32_t other = static_cast<uint32_t>(n) * kSlotU4;  // offset of the second buffer
  uint4* const tx = hop_buf + nxt * kSlotU4 + t;               // the next warp's slot
  const uint4* const rx = hop_buf + r * kSlotU4 + t;           // this warp's slot
  uint32_t bo = 0;                                             // buffer of the current hop
  // this thread's own inputs of the current tile, one 16-byte cell per
  // reduce-scatter step (cell k at mine[k * 32 n]); each thread writes and
  // reads only its own cells
  uint4* const mine = hop_buf + 2 * other + threadIdx.x;
  const uint32_t cells = 32u * static_cast<uint32_t>(n);
  auto wait_cells = [&]() {  // at most n - 1 of this thread's groups in flight
    if constexpr (NR > 0) {
      cp_async_wait_n<NR - 1>();
    } else {
      switch (n - 1) {
        case 1: cp_async_wait_n<1>(); break;
        case 2: cp_async_wait_n<2>(); break;
        case 3: cp_async_wait_n<3>(); break;
        case 4: cp_async_wait_n<4>(); break;
        case 5: cp_async_wait_n<5>(); break;
        case 6: cp_async_wait_n<6>(); break;
        default: cp_async_wait_n<7>(); break;
      }
    }
  };

  // Reduce-scatter step k handles chunk (r - 1 - k) mod n, whose byte offset
  // in a rank's buffer is offs[k]; the last step's chunk is r itself, and
  // all-gather hop j's chunk r - j is offs[j - 1].
  const OFF seg_b = static_cast<OFF>(a.seg * ES);
  OFF offs[KMAX];
  int chunk[KMAX];
  {
    int c = r == 0 ? n - 1 : r - 1;
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      chunk[k] = c;
      offs[k] = static_cast<OFF>(c) * seg_b;
      c = c == 0 ? n - 1 : c - 1;
    }
  }
  // the last step's chunk (rank r's own), kept apart so that a runtime n
  // never indexes the arrays
  const int chunk_last = r;
  const OFF off_last = static_cast<OFF>(r) * seg_b;
  // the vector at element ee of chunk c lies wholly inside the chunk
  auto inside = [&](int c, uint64_t ee) {
    return ee + VN <= a.seg && static_cast<uint64_t>(c) * a.seg + ee + VN <= a.count;
  };
  const uint64_t step_b = static_cast<uint64_t>(gridDim.x) * (TE * ES);  // bytes from a tile to the next
  const char* const in_r = a.in[r];
  const char* in_t = in_r + (blockIdx.x * TE + static_cast<uint64_t>(t) * VN) * ES;  // this lane's vector of chunk 0
  char* out_t = a.out[r] + (blockIdx.x * TE + static_cast<uint64_t>(t) * VN) * ES;

  // copy step k's input of the tile `delta` bytes ahead into cell k: whole
  // (mode 1), or zeros outside the chunk (mode 2); one commit group per cell,
  // empty when there is no next tile (mode 0)
  auto fill = [&](int k, int c, OFF off, int mode, uint64_t delta, uint64_t ee) {
    if (mode == 1 || (mode == 2 && inside(c, ee))) cp_async16(mine + k * cells, in_t + delta + off, 16);
    else if (mode == 2) cp_async16(mine + k * cells, in_r, 0);
    cp_async_commit();
  };

  // the first tile's inputs, in reduce-scatter step order
  {
    const int mode = blockIdx.x < a.full_tiles ? 1 : 2;
    const uint64_t e = blockIdx.x * TE + static_cast<uint64_t>(t) * VN;
#pragma unroll
    for (int k = 0; k < KMAX; ++k)
      if (k < n) fill(k, chunk[k], offs[k], mode, 0, e);
  }

  for (uint64_t tile = blockIdx.x; tile < a.tiles; tile += gridDim.x) {
    const uint64_t nt = tile + gridDim.x;
    const int next = nt >= a.tiles ? 0 : nt < a.full_tiles ? 1 : 2;  // no next tile / whole / checked
    // Cell k is read at step k, between the barriers of hops k and k+1, and
    // refilled with the next tile's step k after the barrier of hop k+1 (so
    // the refill follows the read).  Every thread commits one group per cell,
    // so the group of the cell read at any step has exactly n - 1 newer ones.
    // fast_tag: this tile and the next are full in every chunk (the usual
    // case): no checks and no choice of refill.
    auto hops = [&](auto fast_tag) {
      constexpr bool FAST = decltype(fast_tag)::value;
      const bool full = FAST || tile < a.full_tiles;
      const uint64_t e = tile * TE + static_cast<uint64_t>(t) * VN;
      const uint64_t ne = e + static_cast<uint64_t>(gridDim.x) * TE;
      auto refill = [&](int k, int c, OFF off) {
        if constexpr (FAST) {
          cp_async16(mine + k * cells, in_t + step_b + off, 16);
          cp_async_commit();
        } else {
          fill(k, c, off, next, step_b, ne);
        }
      };
      auto put = [&](int c, OFF off, const uint4& w) {  // this lane's rounded vector of chunk c (at off)
        if (full || inside(c, e)) st16(out_t + off, w);
      };
      // reduce-scatter: N-1 hops of partials; step k adds chunk r-1-k of this rank
      A p[VN];
      {
        wait_cells();
        Vec<DT> w;
        widen16<DT>(mine[0], w);
#pragma unroll
        for (int i = 0; i < VN; ++i) p[i] = w.v[i];
      }
#pragma unroll
      for (int k = 1; k < KMAX; ++k) {
        if (k >= n) break;
        if constexpr (WIRE) {
          Vec<DT> v;
#pragma unroll
          for (int i = 0; i < VN; ++i) v.v[i] = p[i];
          tx[bo] = narrow16<DT>(v);  // the hop's rounding
          __syncthreads();
          widen16<DT>(rx[bo], v);
#pragma unroll
          for (int i = 0; i < VN; ++i) p[i] = v.v[i];
        } else {
#pragma unroll
          for (int q = 0; q < NQ; ++q)
            tx[bo + q * 32] = make_uint4(a_to_bits<DT>(p[4 * q]), a_to_bits<DT>(p[4 * q + 1]),
                                         a_to_bits<DT>(p[4 * q + 2]), a_to_bits<DT>(p[4 * q + 3]));
          __syncthreads();
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            const uint4 x = rx[bo + q * 32];
            p[4 * q] = a_from_bits<DT>(x.x);
            p[4 * q + 1] = a_from_bits<DT>(x.y);
            p[4 * q + 2] = a_from_bits<DT>(x.z);
            p[4 * q + 3] = a_from_bits<DT>(x.w);
          }
        }
        bo = bo == 0 ? other : 0;
        refill(k - 1, chunk[k - 1], offs[k - 1]);  // cell k-1 was read before this barrier
        wait_cells();
        Vec<DT> w;
        widen16<DT>(mine[k * cells], w);
#pragma unroll
        for (int i = 0; i < VN; ++i) p[i] = op_step<OP>(p[i], w.v[i]);
      }
      // the one rounding, on rank r (chunk r is offs[n-1]); the rounded value travels on
      Vec<DT> v;
#pragma unroll
      for (int i = 0; i < VN; ++i) v.v[i] = p[i];
      uint4 w = narrow16<DT>(v);
      put(chunk_last, off_last, w);
      // all-gather: N-1 hops; at hop j chunk r-j (offs[j-1]) arrives, is
      // stored and (but for the last hop) passed on
#pragma unroll
      for (int j = 1; j < KMAX; ++j) {
        if (j >= n) break;
        tx[bo] = w;
        __syncthreads();
        w = rx[bo];
        bo = bo == 0 ? other : 0;
        if (j == 1) refill(n - 1, chunk_last, off_last);  // the last cell, read before this barrier
        put(chunk[j - 1], offs[j - 1], w);
      }
    };
    if (next == 1 && tile < a.full_tiles) hops(std::true_type{});
    else hops(std::false_type{});
    in_t += step_b;
    out_t += step_b;
  }
  cp_async_wait_n<0>();  // nothing of this CTA's is still being copied when it leaves
  if (blockIdx.x == 0 && r == 0) ring_tail<DT, OP, WIRE>(a, t);
}

template <int DT>
static uint64_t ring_cta_tiles(uint64_t seg) {
  const uint64_t per_tile = 32ull * Vec<DT>::kN;
  return std::max<uint64_t>(1, (seg + per_tile - 1) / per_tile);
}

template <int DT, int OP, int MINB, typename OFF, int NR, bool WIRE>
static int launch_ring_cta_t(RingCtaArgs a, cudaStream_t s) {
  constexpr int VN = Vec<DT>::kN;
  constexpr int NQ = WIRE ? 1 : VN / 4;
  const uint64_t per_tile = 32ull * VN;
  a.tiles = ring_cta_tiles<DT>(a.seg);
  // the last chunk is the shortest (possibly empty): a tile is full in every
  // chunk when it is full in that one
  const uint64_t lead = static_cast<uint64_t>(a.n - 1) * a.seg;
  a.full_tiles = a.count > lead ? (a.count - lead) / per_tile : 0;
  const size_t smem = (2ull * NQ + a.n) * a.n * 32 * 16;  // hop slots, then each thread's input cells
  static int smem_set[COLL_MAX_RANKS] = {0};  // per device ordinal: largest limit set so far
  const int st =
      allow_dynamic_smem(reinterpret_cast<const void*>(k_ring_cta<DT, OP, MINB, OFF, NR, WIRE>), smem, smem_set);
  if (st != COLL_OK) return st;
  const uint64_t grid = std::min<uint64_t>(a.tiles, kMaxStreamGrid);  // one CTA per tile, launched in order
  launch_pdl(k_ring_cta<DT, OP, MINB, OFF, NR, WIRE>, dim3(static_cast<unsigned>(grid)), dim3(32 * a.n), smem, s,
             a);
  return launch_status(cudaGetLastError());
}

template <int DT, int OP, bool WIRE>
static int launch_ring_cta_op(const RingCtaArgs& a, cudaStream_t s) {
  // byte offsets within one rank's buffer fit 32 bits below 4 GiB
  const uint64_t span = static_cast<uint64_t>(a.n) * a.seg * Elem<DT>::kSize;
  if (span >= (1ull << 32)) return launch_ring_cta_t<DT, OP, 3, uint64_t, 0, WIRE>(a, s);
  // eight ranks (the workloads' count) get the fully unrolled kernel
  if (a.n == 8) return launch_ring_cta_t<DT, OP, 4, uint32_t, 8, WIRE>(a, s);
  return launch_ring_cta_t<DT, OP, 4, uint32_t, 0, WIRE>(a, s);
}

// Rounding a partial to the storage type changes nothing for fp32 / int32
// (storage = arithmetic type) or for MAX / MIN (the winner's own bits), so
// RING_WIRE runs the fp32 ring's kernels there.
template <int DT, int OP>
static int launch_ring_cta_wire(const RingCtaArgs& a, bool wire, cudaStream_t s) {
  if constexpr ((DT == COLL_BF16 || DT == COLL_FP16) && (OP == COLL_SUM || OP == COLL_PROD)) {
    if (wire) return launch_ring_cta_op<DT, OP, true>(a, s);
  }
  return launch_ring_cta_op<DT, OP, false>(a, s);
}

template <int DT>
static int launch_ring_cta_dt(const RingCtaArgs& a, coll_op_t op, bool wire, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_ring_cta_wire<DT, COLL_SUM>(a, wire, s);
    case COLL_MAX: return launch_ring_cta_wire<DT, COLL_MAX>(a, wire, s);
    case COLL_MIN: return launch_ring_cta_wire<DT, COLL_MIN>(a, wire, s);
    case COLL_PROD: return launch_ring_cta_wire<DT, COLL_PROD>(a, wire, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

bool ring_cta_supported(int n) { return n >= 2 && n <= kRtMaxRanks; }

int launch_ring_cta(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                    bool wire, cudaStream_t s) {
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
  switch (dt) {
    case COLL_BF16: return launch_ring_cta_dt<COLL_BF16>(a, op, wire, s);
    case COLL_FP16: return launch_ring_cta_dt<COLL_FP16>(a, op, wire, s);
    case COLL_FP32: return launch_ring_cta_dt<COLL_FP32>(a, op, wire, s);
    case COLL_INT32: return launch_ring_cta_dt<COLL_INT32>(a, op, wire, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

}  // namespace mvr
