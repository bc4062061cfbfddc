// LL and LL128 packets ("From NCCL Ring LL to PCIe IPC AllReduce", section
// "Traditional LL Protocols"): an LL line is [4 B data | 4 B flag], an LL128
// line is [120 B data | 8 B flag].  The receive side of the page's section
// "Pro5000 ?" reads 16-byte groups and accepts the data only when every flag
// in the group equals the current step; here that check is a validation of
// stream-ordered data, counted into the device status, never a wait.
//
// LL:    one thread per 16-byte group = two lines; a thread of pack reads 16
//        message bytes and writes 32 packet bytes.
// LL128: a warp per group of 4 lines (480 message bytes, 512 packet bytes)
//        when the message is 16-byte aligned, rearranged in shared memory so
//        that both sides move 16-byte units; otherwise eight threads per
//        128-byte line, thread j owning packet bytes [16j, 16j+16) (thread
//        7's chunk carries 8 data bytes and the flag), message-side accesses
//        8 bytes wide since offsets 120L + 16j are only 8-byte aligned.
#include <algorithm>

#include "bulk.cuh"
#include "common.cuh"
#include "internal.h"

namespace mvr {

// CTAs for `units` threads' work: one work item per thread
static unsigned grid_units(uint64_t units) { return static_cast<unsigned>(stream_grid(units, kThreads)); }

// little-endian bytes [off, off+len) of src, zero beyond `bytes`, as a u32/u64
__device__ __forceinline__ uint32_t load_word_tail(const uint8_t* src, uint64_t off, uint64_t bytes) {
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (off + i < bytes) w |= static_cast<uint32_t>(src[off + i]) << (8 * i);
  return w;
}
__device__ __forceinline__ uint2 load8_any(const uint8_t* src, uint64_t off, uint64_t bytes, bool al8) {
  if (off + 8 <= bytes && al8) return ld8(src + off);
  return make_uint2(load_word_tail(src, off, bytes), load_word_tail(src, off + 4, bytes));
}
__device__ __forceinline__ void store_bytes(uint8_t* dst, uint64_t off, uint64_t bytes, uint32_t w) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (off + i < bytes) dst[off + i] = static_cast<uint8_t>(w >> (8 * i));
}
__device__ __forceinline__ void store8_any(uint8_t* dst, uint64_t off, uint64_t bytes, uint2 v, bool al8) {
  if (off + 8 <= bytes && al8) {
    st8(dst + off, v);
  } else {
    store_bytes(dst, off, bytes, v.x);
    store_bytes(dst, off + 4, bytes, v.y);
  }
}

// ------------------------------------------------------------------ LL ----
//
// Every codec kernel serves the n ranks of one call: CTA row blockIdx.y
// takes ranks blockIdx.y, blockIdx.y + gridDim.y, ..., walking each rank's
// message with a grid-stride loop.  The launcher gives every rank its own row
// (gridDim.y = n), so all ranks are in flight at once: measured on one B200
// against one rank after the other (gridDim.y = 1), as fast at 16 MiB per
// rank and 1-2.5% faster at 256 MiB, and 9-21% faster than one launch per
// rank at 16 MiB.  The alignment arguments hold for every rank's pointers.

__device__ __forceinline__ void ll_pack_rank(const uint8_t* __restrict__ src, uint8_t* __restrict__ packed,
                                             uint64_t bytes, uint32_t flag, int src_al16) {
  const uint64_t nlines = (bytes + 3) / 4;
  const uint64_t ngroups = nlines / 4;  // groups of 4 lines = 16 message bytes
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  const uint64_t t0 = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint64_t full = src_al16 ? bytes / 16 : 0;  // groups read with one 16-byte load
  for (uint64_t g = t0; g < ngroups; g += stride) {
    uint4 x;
    if (g < full) {
      x = ld16(src + 16 * g);
    } else {
      x.x = load_word_tail(src, 16 * g, bytes);
      x.y = load_word_tail(src, 16 * g + 4, bytes);
      x.z = load_word_tail(src, 16 * g + 8, bytes);
      x.w = load_word_tail(src, 16 * g + 12, bytes);
    }
    st16(packed + 32 * g, make_uint4(x.x, flag, x.y, flag));
    st16(packed + 32 * g + 16, make_uint4(x.z, flag, x.w, flag));
  }
  for (uint64_t L = 4 * ngroups + t0; L < nlines; L += stride)  // last 1..3 lines
    st8(packed + 8 * L, make_uint2(load_word_tail(src, 4 * L, bytes), flag));
}

__global__ void __launch_bounds__(kThreads) k_ll_pack(const __grid_constant__ CodecArgs a, int src_al16) {
  pdl_wait();
  pdl_trigger();
  for (int r = blockIdx.y; r < a.n; r += gridDim.y) ll_pack_rank(a.in[r], a.out[r], a.bytes, static_cast<uint32_t>(a.step), src_al16);
}

__device__ __forceinline__ int ll_unpack_rank(const uint8_t* __restrict__ packed, uint8_t* __restrict__ dst,
                                              uint64_t bytes, uint32_t flag, int dst_al16) {
  const uint64_t nlines = (bytes + 3) / 4;
  const uint64_t ngroups = nlines / 4;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  const uint64_t t0 = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  int bad = 0;
  for (uint64_t g = t0; g < ngroups; g += stride) {
    const uint4 x0 = ld16(packed + 32 * g);
    const uint4 x1 = ld16(packed + 32 * g + 16);
    bad += (x0.y != flag) + (x0.w != flag) + (x1.y != flag) + (x1.w != flag);
    if (dst_al16 && 16 * g + 16 <= bytes) {
      st16(dst + 16 * g, make_uint4(x0.x, x0.z, x1.x, x1.z));
    } else {
      store_bytes(dst, 16 * g, bytes, x0.x);
      store_bytes(dst, 16 * g + 4, bytes, x0.z);
      store_bytes(dst, 16 * g + 8, bytes, x1.x);
      store_bytes(dst, 16 * g + 12, bytes, x1.z);
    }
  }
  for (uint64_t L = 4 * ngroups + t0; L < nlines; L += stride) {
    const uint2 v = ld8(packed + 8 * L);
    bad += (v.y != flag);
    store_bytes(dst, 4 * L, bytes, v.x);
  }
  return bad;
}

__global__ void __launch_bounds__(kThreads) k_ll_unpack(const __grid_constant__ CodecArgs a, int dst_al16) {
  pdl_wait();
  pdl_trigger();
  int bad = 0;
  for (int r = blockIdx.y; r < a.n; r += gridDim.y)
    bad += ll_unpack_rank(a.in[r], a.out[r], a.bytes, static_cast<uint32_t>(a.step), dst_al16);
  report_warp(a.status, COLL_DEV_FLAG_MISMATCH, bad);
}

// --------------------------------------------------------------- LL128 ----

// A group of 4 lines carries 480 message bytes, a whole number of 16-byte
// units: when the message is 16-byte aligned, a warp moves a group at a
// time with 16-byte accesses on both sides (30 lanes on the message side, 32
// on the packet side), rearranging the bytes in its own 480-byte
// shared-memory buffer; two groups per warp per pass keep two loads in
// flight.  Lines after the last whole group take the 8-threads-per-line code.
constexpr int kGroupBytes = 480;  // 4 lines of payload
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ void ll128_pack_rank(const uint8_t* __restrict__ src, uint8_t* __restrict__ packed,
                                                uint64_t bytes, uint64_t step, int src_al8, int src_al16,
                                                uint8_t (*stage)[2][kGroupBytes]) {
  const uint64_t nlines = (bytes + 119) / 120;
  uint64_t first = 0;  // first line of the 8-threads-per-line part
  if (src_al16) {
    const uint64_t groups = bytes / kGroupBytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int l = lane >> 3, j = lane & 7;  // line of the group, 16-byte chunk of the line
    const uint64_t ws = static_cast<uint64_t>(gridDim.x) * kWarps;
    const uint2 flag = make_uint2(static_cast<uint32_t>(step), static_cast<uint32_t>(step >> 32));
    for (uint64_t g = static_cast<uint64_t>(blockIdx.x) * kWarps + warp; g < groups; g += 2 * ws) {
      const bool two = g + ws < groups;
      uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
      if (lane < 30) {
        x0 = ld16(src + kGroupBytes * g + 16 * lane);
        if (two) x1 = ld16(src + kGroupBytes * (g + ws) + 16 * lane);
        *reinterpret_cast<uint4*>(stage[warp][0] + 16 * lane) = x0;
        *reinterpret_cast<uint4*>(stage[warp][1] + 16 * lane) = x1;
      }
      __syncwarp();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (h == 1 && !two) break;
        const uint8_t* b = stage[warp][h] + 120 * l + 16 * j;
        const uint2 lo = *reinterpret_cast<const uint2*>(b);
        const uint2 hi = j < 7 ? *reinterpret_cast<const uint2*>(b + 8) : flag;
        st16(packed + 512 * (g + h * ws) + 16 * lane, make_uint4(lo.x, lo.y, hi.x, hi.y));
      }
      __syncwarp();
    }
    first = 4 * groups;
  }
  const uint64_t nthreads = (nlines - first) * 8;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t t = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < nthreads; t += stride) {
    const uint64_t L = first + (t >> 3);
    const int j = static_cast<int>(t & 7);
    const uint64_t off = 120 * L + 16 * j;
    const uint2 lo = load8_any(src, off, bytes, src_al8);
    uint2 hi;
    if (j < 7) hi = load8_any(src, off + 8, bytes, src_al8);
    else hi = make_uint2(static_cast<uint32_t>(step), static_cast<uint32_t>(step >> 32));
    st16(packed + 128 * L + 16 * j, make_uint4(lo.x, lo.y, hi.x, hi.y));
  }
}

__global__ void __launch_bounds__(kThreads) k_ll128_pack(const __grid_constant__ CodecArgs a, int src_al8,
                                                         int src_al16) {
  __shared__ __align__(16) uint8_t stage[kWarps][2][kGroupBytes];
  pdl_wait();
  pdl_trigger();
  for (int r = blockIdx.y; r < a.n; r += gridDim.y) ll128_pack_rank(a.in[r], a.out[r], a.bytes, a.step, src_al8, src_al16, stage);
}

__device__ __forceinline__ int ll128_unpack_rank(const uint8_t* __restrict__ packed, uint8_t* __restrict__ dst,
                                                 uint64_t bytes, uint64_t step, int dst_al8, int dst_al16,
                                                 uint8_t (*stage)[2][kGroupBytes]) {
  const uint64_t nlines = (bytes + 119) / 120;
  int bad = 0;
  uint64_t first = 0;
  if (dst_al16) {
    const uint64_t groups = bytes / kGroupBytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int l = lane >> 3, j = lane & 7;
    const uint64_t ws = static_cast<uint64_t>(gridDim.x) * kWarps;
    for (uint64_t g = static_cast<uint64_t>(blockIdx.x) * kWarps + warp; g < groups; g += 2 * ws) {
      const bool two = g + ws < groups;
      const uint4 x0 = ld16(packed + 512 * g + 16 * lane);
      const uint4 x1 = two ? ld16(packed + 512 * (g + ws) + 16 * lane) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (h == 1 && !two) break;
        const uint4 x = h == 0 ? x0 : x1;
        uint8_t* b = stage[warp][h] + 120 * l + 16 * j;
        *reinterpret_cast<uint2*>(b) = make_uint2(x.x, x.y);
        if (j < 7) *reinterpret_cast<uint2*>(b + 8) = make_uint2(x.z, x.w);
        else bad += (static_cast<uint64_t>(x.z) | (static_cast<uint64_t>(x.w) << 32)) != step;
      }
      __syncwarp();
      if (lane < 30) {
        st16(dst + kGroupBytes * g + 16 * lane, *reinterpret_cast<const uint4*>(stage[warp][0] + 16 * lane));
        if (two) st16(dst + kGroupBytes * (g + ws) + 16 * lane, *reinterpret_cast<const uint4*>(stage[warp][1] + 16 * lane));
      }
      __syncwarp();
    }
    first = 4 * groups;
  }
  const uint64_t nthreads = (nlines - first) * 8;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t t = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < nthreads; t += stride) {
    const uint64_t L = first + (t >> 3);
    const int j = static_cast<int>(t & 7);
    const uint4 x = ld16(packed + 128 * L + 16 * j);
    const uint64_t off = 120 * L + 16 * j;
    store8_any(dst, off, bytes, make_uint2(x.x, x.y), dst_al8);
    if (j < 7) {
      store8_any(dst, off + 8, bytes, make_uint2(x.z, x.w), dst_al8);
    } else {
      const uint64_t f = static_cast<uint64_t>(x.z) | (static_cast<uint64_t>(x.w) << 32);
      bad += (f != step);
    }
  }
  return bad;
}

__global__ void __launch_bounds__(kThreads) k_ll128_unpack(const __grid_constant__ CodecArgs a, int dst_al8,
                                                           int dst_al16) {
  __shared__ __align__(16) uint8_t stage[kWarps][2][kGroupBytes];
  pdl_wait();
  pdl_trigger();
  int bad = 0;
  for (int r = blockIdx.y; r < a.n; r += gridDim.y)
    bad += ll128_unpack_rank(a.in[r], a.out[r], a.bytes, a.step, dst_al8, dst_al16, stage);
  report_warp(a.status, COLL_DEV_FLAG_MISMATCH, bad);
}

// ------------------------------------------------ bulk-copy LL pack path ----
//
// LL pack writes twice the bytes it reads, and for long messages bulk stores
// keep more of that in flight than 16-byte stores do (measured at 16 MiB:
// 9.4 us against 11.7 us; unpack and the LL128 codecs measured faster on the
// element kernels, so they stay there).  One warp per CTA bulk-loads 4096
// message bytes into a shared-memory stage, the 32 lanes interleave them
// with the flag into the stage's 8192-byte output buffer, and one lane
// bulk-stores it; STAGES stages overlap loads, rewrites and stores of the
// tiles a CTA takes.  The partial tile at the end goes to k_ll_pack.
constexpr int kPackStages = 4;     // a resident CTA walking many tiles
constexpr int kPackStagesIo = 2;   // a CTA of the in-order grid, one tile per stage
constexpr uint32_t kPackMsg = 4096, kPackPkt = 8192;

template <int STAGES>
__global__ void __launch_bounds__(32) k_ll_pack_tma(const __grid_constant__ CodecArgs a, uint64_t tiles) {
  extern __shared__ __align__(128) unsigned char smem[];  // [stage]{in[kPackMsg], out[kPackPkt]}
  __shared__ __align__(8) uint64_t bar[STAGES];
  constexpr uint32_t kStage = kPackMsg + kPackPkt;
  pdl_wait();
  pdl_trigger();
  const uint32_t flag = static_cast<uint32_t>(a.step);
  const unsigned char* __restrict__ src = a.in[blockIdx.y];  // one rank per CTA row
  unsigned char* __restrict__ packed = a.out[blockIdx.y];
  const uint64_t total = tiles;
  const int lane = threadIdx.x;
  if (lane == 0) {
    for (int st = 0; st < STAGES; ++st) mbar_init(&bar[st], 1);
    fence_barrier_init();
  }
  __syncwarp();
  const uint64_t stride = gridDim.x;
  auto issue = [&](uint64_t t, int st) {  // lane 0
    mbar_arrive_expect_tx(&bar[st], kPackMsg);
    bulk_load(smem + st * kStage, src + t * kPackMsg, kPackMsg, &bar[st]);
  };
  int inflight = 0;
  for (int st = 0; st < STAGES && blockIdx.x + st * stride < total; ++st, ++inflight)
    if (lane == 0) issue(blockIdx.x + st * stride, st);
  int i = 0;
  for (uint64_t t = blockIdx.x; t < total; t += stride, ++i) {
    const int st = i % STAGES;
    const uint32_t par = (i / STAGES) & 1;
    int ok = 1;
    if (lane == 0) {
      ok = mbar_wait_bounded(&bar[st], par) ? 1 : 0;
      bulk_wait_read<STAGES - 1>();  // this stage's previous store has read its output buffer
    }
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (!ok) {
      if (lane == 0) {
        bulk_wait_all();
        for (int k = 1; k < inflight; ++k)
          mbar_wait_bounded(&bar[(i + k) % STAGES], ((i + k) / STAGES) & 1);
      }
      return;
    }
    mbar_try_wait(&bar[st], par);  // completed: every lane acquires the loaded tile itself
    --inflight;
    const unsigned char* in = smem + st * kStage;
    unsigned char* out = smem + st * kStage + kPackMsg;
    for (int c = lane; c < static_cast<int>(kPackMsg / 16); c += 32) {  // 16 bytes -> {d, f, d, f} {d, f, d, f}
      const uint4 x = *reinterpret_cast<const uint4*>(in + 16 * c);
      *reinterpret_cast<uint4*>(out + 32 * c) = make_uint4(x.x, flag, x.y, flag);
      *reinterpret_cast<uint4*>(out + 32 * c + 16) = make_uint4(x.z, flag, x.w, flag);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the rewrite, visible to the bulk copies
    __syncwarp();
    if (lane == 0) {
      bulk_store(packed + t * kPackPkt, out, kPackPkt);
      bulk_commit();
      const uint64_t nxt = t + STAGES * stride;
      if (nxt < total) {
        issue(nxt, st);
        ++inflight;
      }
    }
    inflight = __shfl_sync(0xFFFFFFFFu, inflight, 0);
  }
  if (lane == 0) bulk_wait_all();
}

template <int STAGES>
static int launch_pack_tma(const CodecArgs& a, unsigned gx, uint64_t tiles, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(STAGES) * (kPackMsg + kPackPkt);
  static int smem_set[COLL_MAX_RANKS] = {0};  // per device ordinal: largest limit set so far
  const int ok = allow_dynamic_smem(reinterpret_cast<const void*>(k_ll_pack_tma<STAGES>), smem, smem_set);
  if (ok != COLL_OK) return ok;
  launch_pdl(k_ll_pack_tma<STAGES>, dim3(gx, a.n), dim3(32), smem, s, a, tiles);
  return launch_status(cudaGetLastError());
}

// The codec grid for n ranks of `units` work items each: one CTA row per
// rank, about eight work items per thread, the CTAs launched in order.  The
// warps walk several line groups each (for LL128, two per pass), so one item
// per thread (20-60% slower) gives a CTA too little work, and a resident grid
// walking the data with a stride measured 7-14% slower for the LL128 codecs
// at 16 and 256 MiB per rank (LL128 pack at 8 x 256 MiB: 757 -> 651 us).
static dim3 codec_grid(uint64_t units, int n) {
  constexpr uint64_t kItemsPerThread = 8;
  return dim3(static_cast<unsigned>(stream_grid((units + kItemsPerThread - 1) / kItemsPerThread, kThreads)),
              static_cast<unsigned>(n));
}

// every message pointer's low bits, and every packet pointer's
static void codec_bits(const CodecArgs& a, uintptr_t& msg, uintptr_t& pkt, bool pack) {
  msg = pkt = 0;
  for (int r = 0; r < a.n; ++r) {
    msg |= reinterpret_cast<uintptr_t>(pack ? static_cast<const void*>(a.in[r]) : static_cast<const void*>(a.out[r]));
    pkt |= reinterpret_cast<uintptr_t>(pack ? static_cast<const void*>(a.out[r]) : static_cast<const void*>(a.in[r]));
  }
}

int launch_ll_pack(const CodecArgs& a0, int proto, cudaStream_t s) {
  if (a0.bytes == 0 || a0.n < 1) return COLL_OK;
  CodecArgs a = a0;
  uintptr_t msg, pkt;
  codec_bits(a, msg, pkt, true);
  const dim3 block(kThreads);
  if (proto == COLL_PROTO_LL && ((msg | pkt) & 15) == 0) {
    // whole tiles through the bulk-copy path from 4 tiles per resident CTA up
    // (4 x 48 KB of stages per SM, shared by the ranks' CTA rows), the rest
    // below.  From 8 tiles per resident CTA up, one CTA per 2 tiles of a
    // rank with 2 stages (24 KB, so 9 CTAs fit on an SM), launched in order:
    // measured faster than a resident grid walking the tiles (8 x 256 MiB:
    // 935 against 1081 us; 4 tiles and 4 stages per CTA 977 us).  Below that
    // the in-order grid would end on a partial second wave, and the resident
    // grid with 4 stages is faster (one rank of 16 MiB: 9.35 against 10.24 us).
    const uint64_t resident = std::max<uint64_t>(1, static_cast<uint64_t>(num_sms()) * 4 / a.n);
    const uint64_t tiles = a.bytes / kPackMsg;  // per rank
    if (tiles >= 4 * resident) {
      const int st = tiles < 8 * resident
                         ? launch_pack_tma<kPackStages>(a, static_cast<unsigned>(resident), tiles, s)
                         : launch_pack_tma<kPackStagesIo>(a, static_cast<unsigned>(stream_grid(tiles, kPackStagesIo)),
                                                          tiles, s);
      if (st != COLL_OK) return st;
      for (int r = 0; r < a.n; ++r) {
        a.in[r] += tiles * kPackMsg;
        a.out[r] += tiles * kPackPkt;
      }
      a.bytes -= tiles * kPackMsg;
      if (a.bytes == 0) return COLL_OK;
    }
  }
  if (proto == COLL_PROTO_LL) {
    const uint64_t nlines = (a.bytes + 3) / 4;
    launch_pdl(k_ll_pack, codec_grid(nlines / 4 + 1, a.n), block, 0, s, a,
               static_cast<int>((msg & 15) == 0));
  } else {
    const uint64_t nlines = (a.bytes + 119) / 120;
    launch_pdl(k_ll128_pack, codec_grid(nlines * 8, a.n), block, 0, s, a,
               static_cast<int>((msg & 7) == 0), static_cast<int>(((msg | pkt) & 15) == 0));
  }
  return launch_status(cudaGetLastError());
}

int launch_ll_unpack(const CodecArgs& a, int proto, cudaStream_t s) {
  if (a.bytes == 0 || a.n < 1) return COLL_OK;
  uintptr_t msg, pkt;
  codec_bits(a, msg, pkt, false);
  const dim3 block(kThreads);
  if (proto == COLL_PROTO_LL) {
    const uint64_t nlines = (a.bytes + 3) / 4;
    launch_pdl(k_ll_unpack, codec_grid(nlines / 4 + 1, a.n), block, 0, s, a,
               static_cast<int>((msg & 15) == 0));
  } else {
    const uint64_t nlines = (a.bytes + 119) / 120;
    launch_pdl(k_ll128_unpack, codec_grid(nlines * 8, a.n), block, 0, s, a,
               static_cast<int>((msg & 7) == 0), static_cast<int>(((msg | pkt) & 15) == 0));
  }
  return launch_status(cudaGetLastError());
}

// ------------------------------------------------- packetised all-reduce ----

// the elements of one 32-bit data word, zeroed at and beyond `limit`
template <int DT, int OP>
struct WordOps {
  static constexpr int kE = 4 / Elem<DT>::kSize;
  using A = typename Elem<DT>::A;
  static __device__ __forceinline__ void widen(uint32_t w, A (&o)[kE]) {
    if constexpr (kE == 2) {
      o[0] = widen1<DT>(static_cast<uint16_t>(w & 0xFFFFu));
      o[1] = widen1<DT>(static_cast<uint16_t>(w >> 16));
    } else {
      o[0] = widen1<DT>(w);
    }
  }
  static __device__ __forceinline__ void step(A (&acc)[kE], uint32_t w) {
    A v[kE];
    widen(w, v);
#pragma unroll
    for (int i = 0; i < kE; ++i) acc[i] = op_step<OP>(acc[i], v[i]);
  }
  // elem0: element index of the word's first element; count: payload elements
  static __device__ __forceinline__ uint32_t narrow(const A (&acc)[kE], uint64_t elem0, uint64_t count) {
    if constexpr (kE == 2) {
      const uint32_t lo = elem0 < count ? narrow1<DT>(acc[0]) : 0u;
      const uint32_t hi = elem0 + 1 < count ? narrow1<DT>(acc[1]) : 0u;
      return lo | (hi << 16);
    } else {
      return elem0 < count ? narrow1<DT>(acc[0]) : 0u;
    }
  }
};

// LL: thread = one 8-byte line per rank when `single`, else two lines (16 B)
template <int DT, int OP, int NR>  // NR: ranks known at compile time (0 = runtime): all NR loads issued at once
__global__ void __launch_bounds__(kThreads) k_ar_ll(const __grid_constant__ PackedReduceArgs a) {
  pdl_wait();
  pdl_trigger();
  using W = WordOps<DT, OP>;
  using A = typename Elem<DT>::A;
  constexpr int kE = W::kE;
  const uint32_t flag = static_cast<uint32_t>(a.step);
  const uint64_t count = a.payload_bytes / Elem<DT>::kSize;
  const uint64_t ngroups = a.nlines / 2;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  const uint64_t t0 = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  int bad = 0;
  for (uint64_t g = t0; g < ngroups; g += stride) {
    A acc0[kE], acc1[kE];
    if constexpr (NR > 0) {
      uint4 xs[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) xs[r] = ld16(a.in[r] + 16 * g);
      W::widen(xs[0].x, acc0);
      W::widen(xs[0].z, acc1);
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        bad += (xs[r].y != flag) + (xs[r].w != flag);
        if (r > 0) {
          W::step(acc0, xs[r].x);
          W::step(acc1, xs[r].z);
        }
      }
    } else {
      uint4 x = ld16(a.in[0] + 16 * g);
      bad += (x.y != flag) + (x.w != flag);
      W::widen(x.x, acc0);
      W::widen(x.z, acc1);
      for (int r = 1; r < a.n; ++r) {
        x = ld16(a.in[r] + 16 * g);
        bad += (x.y != flag) + (x.w != flag);
        W::step(acc0, x.x);
        W::step(acc1, x.z);
      }
    }
    const uint64_t e0 = 2 * g * kE;  // first element of line 2g
    const uint4 o = make_uint4(W::narrow(acc0, e0, count), flag, W::narrow(acc1, e0 + kE, count), flag);
    for (int q = 0; q < a.n; ++q) st16(a.out[q] + 16 * g, o);
  }
  if ((a.nlines & 1) && t0 == 0) {  // odd last line
    const uint64_t L = a.nlines - 1;
    A acc[kE];
    uint2 x = ld8(a.in[0] + 8 * L);
    bad += (x.y != flag);
    W::widen(x.x, acc);
    for (int r = 1; r < a.n; ++r) {
      x = ld8(a.in[r] + 8 * L);
      bad += (x.y != flag);
      W::step(acc, x.x);
    }
    const uint2 o = make_uint2(W::narrow(acc, L * kE, count), flag);
    for (int q = 0; q < a.n; ++q) st8(a.out[q] + 8 * L, o);
  }
  report_warp(a.status, COLL_DEV_FLAG_MISMATCH, bad);
}

// LL128: eight threads per line, thread j owns packet bytes [16j, 16j+16)
template <int DT, int OP, int NR>
__global__ void __launch_bounds__(kThreads) k_ar_ll128(const __grid_constant__ PackedReduceArgs a) {
  pdl_wait();
  pdl_trigger();
  using W = WordOps<DT, OP>;
  using A = typename Elem<DT>::A;
  constexpr int kE = W::kE;
  constexpr int ES = Elem<DT>::kSize;
  const uint64_t count = a.payload_bytes / ES;
  const uint64_t nthreads = a.nlines * 8;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  int bad = 0;
  for (uint64_t t = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < nthreads; t += stride) {
    const uint64_t L = t >> 3;
    const int j = static_cast<int>(t & 7);
    const uint64_t poff = 128 * L + 16 * j;
    const uint64_t e0 = (120 * L + 16 * j) / ES;  // first element of this chunk
    A acc[4][kE];
    auto first = [&](const uint4& x) {
      if (j == 7) bad += ((static_cast<uint64_t>(x.z) | (static_cast<uint64_t>(x.w) << 32)) != a.step);
      W::widen(x.x, acc[0]);
      W::widen(x.y, acc[1]);
      W::widen(x.z, acc[2]);
      W::widen(x.w, acc[3]);
    };
    auto next = [&](const uint4& x) {
      if (j == 7) bad += ((static_cast<uint64_t>(x.z) | (static_cast<uint64_t>(x.w) << 32)) != a.step);
      W::step(acc[0], x.x);
      W::step(acc[1], x.y);
      W::step(acc[2], x.z);
      W::step(acc[3], x.w);
    };
    if constexpr (NR > 0) {
      uint4 xs[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) xs[r] = ld16(a.in[r] + poff);
      first(xs[0]);
#pragma unroll
      for (int r = 1; r < NR; ++r) next(xs[r]);
    } else {
      first(ld16(a.in[0] + poff));
      for (int r = 1; r < a.n; ++r) next(ld16(a.in[r] + poff));
    }
    uint4 o;
    o.x = W::narrow(acc[0], e0, count);
    o.y = W::narrow(acc[1], e0 + kE, count);
    if (j < 7) {
      o.z = W::narrow(acc[2], e0 + 2 * kE, count);
      o.w = W::narrow(acc[3], e0 + 3 * kE, count);
    } else {
      o.z = static_cast<uint32_t>(a.step);
      o.w = static_cast<uint32_t>(a.step >> 32);
    }
    for (int q = 0; q < a.n; ++q) st16(a.out[q] + poff, o);
  }
  report_warp(a.status, COLL_DEV_FLAG_MISMATCH, bad);
}

template <int DT, int OP>
static int launch_ar_packed_t(const PackedReduceArgs& a, int proto, cudaStream_t s) {
  // the 8-rank sum (the workloads' rank count) issues its eight loads at once
  const bool eight = a.n == 8 && OP == COLL_SUM;
  if (proto == COLL_PROTO_LL) {
    if (eight)
      launch_pdl(k_ar_ll<DT, OP, 8>, dim3(grid_units(a.nlines / 2 + 1)),
                 dim3(kThreads), 0, s, a);
    else
      launch_pdl(k_ar_ll<DT, OP, 0>, dim3(grid_units(a.nlines / 2 + 1)),
                 dim3(kThreads), 0, s, a);
  } else {
    if (eight)
      launch_pdl(k_ar_ll128<DT, OP, 8>,
                 dim3(grid_units(a.nlines * 8)), dim3(kThreads), 0,
                 s, a);
    else
      launch_pdl(k_ar_ll128<DT, OP, 0>,
                 dim3(grid_units(a.nlines * 8)), dim3(kThreads), 0,
                 s, a);
  }
  return launch_status(cudaGetLastError());
}

template <int DT>
static int launch_ar_packed_dt(const PackedReduceArgs& a, coll_op_t op, int proto, cudaStream_t s) {
  switch (op) {
    case COLL_SUM: return launch_ar_packed_t<DT, COLL_SUM>(a, proto, s);
    case COLL_MAX: return launch_ar_packed_t<DT, COLL_MAX>(a, proto, s);
    case COLL_MIN: return launch_ar_packed_t<DT, COLL_MIN>(a, proto, s);
    case COLL_PROD: return launch_ar_packed_t<DT, COLL_PROD>(a, proto, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

int launch_all_reduce_packed(const PackedReduceArgs& a, coll_dtype_t dt, coll_op_t op, int proto, cudaStream_t s) {
  if (a.nlines == 0) return COLL_OK;
  switch (dt) {
    case COLL_BF16: return launch_ar_packed_dt<COLL_BF16>(a, op, proto, s);
    case COLL_FP16: return launch_ar_packed_dt<COLL_FP16>(a, op, proto, s);
    case COLL_FP32: return launch_ar_packed_dt<COLL_FP32>(a, op, proto, s);
    case COLL_INT32: return launch_ar_packed_dt<COLL_INT32>(a, op, proto, s);
  }
  return COLL_ERR_UNSUPPORTED;
}

}  // namespace mvr
