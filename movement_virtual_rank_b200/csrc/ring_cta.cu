// Ring all-reduce with the virtual ranks as warps of one CTA: the hop from
// rank r to rank r+1 is a store into a shared-memory slot of the same SM,
// and every hop of the ring is one CTA-wide barrier.
//
// The schedule, chunk order, fp32 partials and the single rounding are those
// of coll_all_reduce(RING) (TP communication essay; NCCL's ring kernel named
// in "From NCCL Ring LL to PCIe IPC AllReduce"), so the result is
// bit-identical.  A CTA holds all N ranks, one warp each (lane t of warp r
// plays rank r for U 16-byte vectors of every chunk of a tile of 32 x VN x U
// elements); the CTAs of the grid walk the tiles with a stride.
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
// Inputs are prefetched one tile ahead in registers: the vector of step k of
// the next tile is loaded as soon as step k of this tile has used its own.
// Tiles that are full in every chunk (those that end within the last chunk,
// the shortest) take a path with no bounds checks; the others check each
// vector against its chunk's end and handle a ragged vector element by
// element.  Nothing leaves the SM but the loads of inputs and the stores of
// outputs.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace mvr {

constexpr int kRtMaxRanks = 8;

struct RingCtaArgs {
  const char* in[kMaxRanks];
  char* out[kMaxRanks];
  uint64_t count, seg, tiles;
  uint64_t full_tiles;  // tiles [0, full_tiles) are full in every chunk
  int n;
};

template <int DT, int OP, int U, int MINB>
__global__ void __launch_bounds__(kRtMaxRanks * 32, MINB) k_ring_cta(const __grid_constant__ RingCtaArgs a) {
  using A = typename Elem<DT>::A;
  using S = typename Elem<DT>::S;
  constexpr int VN = Vec<DT>::kN;  // elements per 16-byte vector
  constexpr int NQ = VN / 4;       // 16-byte pieces of a vector's fp32 / int32 partials
  constexpr int ES = Elem<DT>::kSize;
  constexpr uint64_t TE = 32ull * VN * U;     // elements of one chunk per tile
  constexpr uint32_t kSlotU4 = 32 * U * NQ;   // one warp's slot, in 16-byte units
  extern __shared__ __align__(16) uint4 hop_buf[];  // [2 buffers][N receiving warps][kSlotU4]
  const int n = a.n;
  const int r = static_cast<int>(threadIdx.x >> 5);
  const int t = static_cast<int>(threadIdx.x & 31);
  pdl_wait();
  pdl_trigger();

  const int nxt = r + 1 == n ? 0 : r + 1;
  const uint32_t other = static_cast<uint32_t>(n) * kSlotU4;  // offset of the second buffer
  uint4* const tx = hop_buf + nxt * kSlotU4 + t;               // the next warp's slot
  const uint4* const rx = hop_buf + r * kSlotU4 + t;           // this warp's slot
  uint32_t bo = 0;                                             // buffer of the current hop

  // chunk c of a rank starts c * seg elements in; reduce-scatter step k
  // handles chunk (r - 1 - k) mod n, all-gather hop j chunk (r - j) mod n:
  // both walk the chunks downwards, wrapping from 0 to n - 1
  const int64_t seg_b = static_cast<int64_t>(a.seg) * ES;
  const int64_t top_b = static_cast<int64_t>(n - 1) * seg_b;
  const int c0 = r == 0 ? n - 1 : r - 1;
  const int64_t off0 = static_cast<int64_t>(c0) * seg_b;
  const int64_t off_r = static_cast<int64_t>(r) * seg_b;
  auto down = [&](int64_t off) { return off == 0 ? top_b : off - seg_b; };
  auto dec = [&](int c) { return c == 0 ? n - 1 : c - 1; };
  const char* const in_r = a.in[r];
  char* const out_r = a.out[r];
  auto chunk_end = [&](int c) { return min(static_cast<uint64_t>(c) * a.seg + a.seg, a.count); };
  auto vec_elem = [&](uint64_t tile, int u) { return tile * TE + static_cast<uint64_t>(u * 32 + t) * VN; };

  auto to_bits = [](A x) -> uint32_t {
    if constexpr (std::is_same<A, float>::value) return __float_as_uint(x);
    else return static_cast<uint32_t>(x);
  };
  auto from_bits = [](uint32_t w) -> A {
    if constexpr (std::is_same<A, float>::value) return __uint_as_float(w);
    else return static_cast<A>(static_cast<int32_t>(w));
  };

  // this lane's vectors of chunk c (byte offset off) in `tile`; zero where a
  // vector is not wholly inside the chunk or the tile is past the end
  auto load = [&](uint64_t tile, int c, int64_t off, uint4 (&dst)[U]) {
    const bool full = tile < a.full_tiles;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint64_t e = vec_elem(tile, u);
      dst[u] = make_uint4(0, 0, 0, 0);
      if (tile < a.tiles && (full || static_cast<uint64_t>(c) * a.seg + e + VN <= chunk_end(c)))
        dst[u] = ld16(in_r + off + static_cast<int64_t>(e * ES));
    }
  };

  const uint64_t G = gridDim.x;
  uint4 pre[kRtMaxRanks][U];
  {
    int c = c0;
    int64_t off = off0;
#pragma unroll
    for (int k = 0; k < kRtMaxRanks; ++k) {
      if (k < n) {
        load(blockIdx.x, c, off, pre[k]);
        off = down(off);
        c = dec(c);
      }
    }
  }

  for (uint64_t tile = blockIdx.x; tile < a.tiles; tile += G) {
    const uint64_t nt = tile + G;
    const bool full = tile < a.full_tiles;

    // own values of reduce-scatter step k (chunk c at byte offset off): the
    // prefetched vector, or a ragged vector element by element; then the
    // same step of the next tile is fetched into the freed registers
    auto own = [&](uint4 (&pk)[U], int c, int64_t off, A (&v)[U][VN]) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint64_t e = vec_elem(tile, u);
        const uint64_t gi = static_cast<uint64_t>(c) * a.seg + e;
        if (full || gi + VN <= chunk_end(c)) {
          Vec<DT> w;
          widen16<DT>(pk[u], w);
#pragma unroll
          for (int i = 0; i < VN; ++i) v[u][i] = w.v[i];
        } else {
          const uint64_t end = chunk_end(c);
#pragma unroll
          for (int i = 0; i < VN; ++i)
            v[u][i] = gi + i < end ? widen1<DT>(*reinterpret_cast<const S*>(in_r + off + (e + i) * ES)) : A(0);
        }
      }
      load(nt, c, off, pk);
    };
    // store this lane's rounded vectors of chunk c (byte offset off)
    auto put = [&](int c, int64_t off, const uint4 (&w)[U]) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint64_t e = vec_elem(tile, u);
        char* const dst = out_r + off + e * ES;
        if (full) {
          st16(dst, w[u]);
          continue;
        }
        const uint64_t gi = static_cast<uint64_t>(c) * a.seg + e;
        const uint64_t end = chunk_end(c);
        if (gi + VN <= end) {
          st16(dst, w[u]);
        } else {
          const S* sv = reinterpret_cast<const S*>(&w[u]);
#pragma unroll
          for (int i = 0; i < VN; ++i)
            if (gi + i < end) *reinterpret_cast<S*>(dst + i * ES) = sv[i];
        }
      }
    };

    // reduce-scatter: N-1 hops of partials; chunk r is complete at the end
    A p[U][VN];
    int c = c0;
    int64_t off = off0;
    own(pre[0], c, off, p);
#pragma unroll
    for (int k = 1; k < kRtMaxRanks; ++k) {
      if (k >= n) break;
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          tx[bo + (u * NQ + q) * 32] = make_uint4(to_bits(p[u][4 * q]), to_bits(p[u][4 * q + 1]),
                                                  to_bits(p[u][4 * q + 2]), to_bits(p[u][4 * q + 3]));
      __syncthreads();
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const uint4 x = rx[bo + (u * NQ + q) * 32];
          p[u][4 * q] = from_bits(x.x);
          p[u][4 * q + 1] = from_bits(x.y);
          p[u][4 * q + 2] = from_bits(x.z);
          p[u][4 * q + 3] = from_bits(x.w);
        }
      bo = bo == 0 ? other : 0;
      c = dec(c);
      off = down(off);
      A x[U][VN];
      own(pre[k], c, off, x);
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int i = 0; i < VN; ++i) p[u][i] = op_step<OP>(p[u][i], x[u][i]);
    }
    // the one rounding, on rank r (c == r); the rounded value travels on
    uint4 w[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      Vec<DT> v;
#pragma unroll
      for (int i = 0; i < VN; ++i) v.v[i] = p[u][i];
      w[u] = narrow16<DT>(v);
    }
    put(r, off_r, w);

    // all-gather: N-1 hops; at hop j chunk r - j arrives, is stored and
    // (but for the last hop) passed on
    int cj = r;
    int64_t offj = off_r;
    for (int j = 1; j < n; ++j) {
#pragma unroll
      for (int u = 0; u < U; ++u) tx[bo + u * 32] = w[u];
      __syncthreads();
#pragma unroll
      for (int u = 0; u < U; ++u) w[u] = rx[bo + u * 32];
      bo = bo == 0 ? other : 0;
      cj = dec(cj);
      offj = down(offj);
      put(cj, offj, w);
    }
  }
}

template <int DT, int OP, int U, int MINB>
static int launch_ring_cta_t(RingCtaArgs a, cudaStream_t s) {
  constexpr int VN = Vec<DT>::kN;
  constexpr int NQ = VN / 4;
  const uint64_t per_tile = 32ull * VN * U;
  a.tiles = std::max<uint64_t>(1, (a.seg + per_tile - 1) / per_tile);
  // the last chunk is the shortest (possibly empty): a tile is full in every
  // chunk when it is full in that one
  const uint64_t lead = static_cast<uint64_t>(a.n - 1) * a.seg;
  a.full_tiles = a.count > lead ? (a.count - lead) / per_tile : 0;
  const size_t smem = 2ull * a.n * 32 * U * NQ * 16;
  static int smem_set[COLL_MAX_RANKS] = {0};  // per device ordinal: largest limit set so far
  const int st = allow_dynamic_smem(reinterpret_cast<const void*>(k_ring_cta<DT, OP, U, MINB>), smem, smem_set);
  if (st != COLL_OK) return st;
  const uint64_t grid = std::min<uint64_t>(a.tiles, static_cast<uint64_t>(num_sms()) * MINB);
  launch_pdl(k_ring_cta<DT, OP, U, MINB>, dim3(static_cast<unsigned>(grid)), dim3(32 * a.n), smem, s, a);
  return launch_status(cudaGetLastError());
}

template <int DT>
static int launch_ring_cta_dt(const RingCtaArgs& a, coll_op_t op, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_ring_cta_t<DT, COLL_SUM, 1, 3>(a, s);
    case COLL_MAX: return launch_ring_cta_t<DT, COLL_MAX, 1, 3>(a, s);
    case COLL_MIN: return launch_ring_cta_t<DT, COLL_MIN, 1, 3>(a, s);
    case COLL_PROD: return launch_ring_cta_t<DT, COLL_PROD, 1, 3>(a, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

bool ring_cta_supported(int n) { return n >= 2 && n <= kRtMaxRanks; }

int launch_ring_cta(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                    int* status, cudaStream_t s) {
  (void)status;  // nothing in this form waits, so it never raises a status
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
    case COLL_BF16: return launch_ring_cta_dt<COLL_BF16>(a, op, s);
    case COLL_FP16: return launch_ring_cta_dt<COLL_FP16>(a, op, s);
    case COLL_FP32: return launch_ring_cta_dt<COLL_FP32>(a, op, s);
    case COLL_INT32: return launch_ring_cta_dt<COLL_INT32>(a, op, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

}  // namespace mvr
