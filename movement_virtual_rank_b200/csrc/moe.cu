// MoE expert-parallel dispatch and combine over virtual ranks (vLLM
// collectives tutorial, section 8.4: tokens go to the rank that holds their
// expert, results come back by original token ownership; section 8.2: the
// per-pair lengths differ, so the exchange is an all-to-all-v).
//
// Route (three launches, deterministic -- no result depends on atomics'
// order).  A bucket is an expert (one row per (token, expert) pair) or, for
// the route deduplicated per (token, destination rank) that the tutorial
// names in 8.5.1, a destination rank (one row per (token, rank)):
//  1. k_moe_count  per (source, tile of 256 tokens): a token x bucket bitmap
//                  in shared memory gives every pair its rank among the
//                  tile's tokens in the same bucket (popcount of the lower
//                  tokens' bits) and every bucket its count in the tile; a
//                  token's second expert on one rank sets the same bit again.
//  2. k_moe_scan   per source: exclusive scan of the counts in (bucket, tile)
//                  order = the send order (destination, expert, token), or
//                  (destination, token); the per-destination send counts and
//                  displacements fall out.
//  3. k_moe_pos    per (source, tile): receive displacements (sum over lower
//                  sources, tutorial 8.1's [from 0, from 1, ...]) plus the
//                  pair's send offset within its destination block.
// Dispatch: one CTA per token row at a time reads the row once and writes it
// to its topk receive rows, once per distinct row (a deduplicated route gives
// the choices of a token that share a rank the same row).  Combine: one CTA per output row reads the topk
// expert rows and forms acc = fl32(w0*y0), acc = fl32(acc + fl32(wk*yk)).
#include <algorithm>

#include "bulk.cuh"
#include "common.cuh"
#include "internal.h"

namespace mvr {

constexpr int kTile = 256;       // tokens per route tile (one per thread)
constexpr int kWords = kTile / 32;
constexpr int kMoveThreads = 128;
constexpr int kMaxTopk = 32;

size_t moe_route_workspace(int n, int tokens, int topk, int n_experts) {
  (void)topk;
  const size_t tiles = (static_cast<size_t>(tokens) + kTile - 1) / kTile;
  const size_t cells = static_cast<size_t>(n) * n_experts * std::max<size_t>(tiles, 1);
  const size_t a = (cells * sizeof(int32_t) + 255) / 256 * 256;
  const size_t b = (cells * sizeof(int64_t) + 255) / 256 * 256;
  return a + b;
}

__global__ void __launch_bounds__(kTile) k_moe_count(const __grid_constant__ MoeRouteArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint32_t bits[];  // [buckets][kWords]
  const int s = blockIdx.x / a.tiles;
  const int tile = blockIdx.x % a.tiles;
  const int E = a.n_experts;
  const int B = a.buckets;
  const int epr = E / a.n;
  for (int i = threadIdx.x; i < B * kWords; i += blockDim.x) bits[i] = 0;
  __syncthreads();
  const int t = threadIdx.x;
  const int tok = tile * kTile + t;
  const bool live = tok < a.tokens;
  const int32_t* ids = a.ids[s] + static_cast<int64_t>(tok) * a.topk;
  const uint32_t me = 1u << (t & 31);
  int bad = 0;
  if (live) {
    for (int k = 0; k < a.topk; ++k) {
      const int e = ids[k];
      if (e < 0 || e >= E) {
        ++bad;
        continue;
      }
      const int b = a.dedup ? e / epr : e;
      const uint32_t old = atomicOr(&bits[b * kWords + (t >> 5)], me);
      if (a.dedup) {
        for (int k2 = 0; k2 < k; ++k2) bad += ids[k2] == e;  // the same expert twice for one token
      } else if (old & me) {
        ++bad;
      }
    }
  }
  __syncthreads();
  if (live) {
    int32_t* pos = a.pos[s] + static_cast<int64_t>(tok) * a.topk;
    for (int k = 0; k < a.topk; ++k) {
      const int e = ids[k];
      if (e < 0 || e >= E) continue;
      const uint32_t* row = bits + (a.dedup ? e / epr : e) * kWords;
      int rank = __popc(row[t >> 5] & (me - 1u));
      for (int w = 0; w < (t >> 5); ++w) rank += __popc(row[w]);
      pos[k] = rank;  // local rank; k_moe_pos adds the block offsets
    }
  }
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWords; ++w) c += __popc(bits[b * kWords + w]);
    a.tile_cnt[(static_cast<int64_t>(s) * B + b) * a.tiles + tile] = c;
  }
  report_warp(a.status, COLL_DEV_BAD_ROUTE, bad);
}

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) k_moe_scan(const __grid_constant__ MoeRouteArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ int64_t warp_sums[kScanThreads / 32];
  const int s = blockIdx.x;
  const int64_t m = static_cast<int64_t>(a.buckets) * a.tiles;  // cells of this source
  const int32_t* cnt = a.tile_cnt + s * m;
  int64_t* base = a.tile_base + s * m;
  const int64_t per = (m + kScanThreads - 1) / kScanThreads;
  const int64_t lo = min(m, per * static_cast<int64_t>(threadIdx.x));
  const int64_t hi = min(m, lo + per);
  int64_t sum = 0;
  for (int64_t i = lo; i < hi; ++i) sum += cnt[i];
  // block-wide exclusive scan of the per-thread sums
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int64_t w = warp_sums[lane];
    int64_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t v = __shfl_up_sync(0xFFFFFFFFu, wi, o);
      if (lane >= o) wi += v;
    }
    warp_sums[lane] = wi - w;  // exclusive over warps
  }
  __syncthreads();
  int64_t run = warp_sums[warp] + incl - sum;
  for (int64_t i = lo; i < hi; ++i) {
    base[i] = run;
    run += cnt[i];
  }
  __syncthreads();
  // per destination: buckets [d*bpr, (d+1)*bpr) are cells [d*bpr*tiles, (d+1)*bpr*tiles)
  const int bpr = a.bpr;
  if (threadIdx.x < a.n) {
    const int d = threadIdx.x;
    const int64_t c0 = static_cast<int64_t>(d) * bpr * a.tiles;
    const int64_t c1 = c0 + static_cast<int64_t>(bpr) * a.tiles;
    // base[c] is visible: written above by this block, ordered by __syncthreads
    const int64_t b0 = c0 < m ? base[c0] : 0;
    int64_t total = 0;
    if (m > 0) total = base[m - 1] + cnt[m - 1];
    const int64_t b1 = c1 < m ? base[c1] : total;
    a.send_displs[s * a.n + d] = b0;
    a.send_counts[s * a.n + d] = b1 - b0;
  }
}

__global__ void __launch_bounds__(kTile) k_moe_pos(const __grid_constant__ MoeRouteArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ int64_t rdispl[kMaxRanks];  // recv_displs[d][s] for this block's s
  __shared__ int64_t sdispl[kMaxRanks];  // send_displs[s][d]
  const int s = blockIdx.x / a.tiles;
  const int tile = blockIdx.x % a.tiles;
  const int n = a.n;
  if (threadIdx.x < n) {
    const int d = threadIdx.x;
    int64_t acc = 0;
    for (int q = 0; q < s; ++q) acc += a.send_counts[q * n + d];
    rdispl[d] = acc;
    sdispl[d] = a.send_displs[s * n + d];
  }
  if (blockIdx.x == 0) {  // the full receive-displacement matrix, [d][s]
    for (int i = threadIdx.x; i < n * n; i += blockDim.x) {
      const int d = i / n, q = i % n;
      int64_t acc = 0;
      for (int p = 0; p < q; ++p) acc += a.send_counts[p * n + d];
      a.recv_displs[d * n + q] = acc;
    }
  }
  __syncthreads();
  const int tok = tile * kTile + threadIdx.x;
  if (tok >= a.tokens) return;
  const int E = a.n_experts;
  const int epr = E / n;
  const int32_t* ids = a.ids[s] + static_cast<int64_t>(tok) * a.topk;
  int32_t* pos = a.pos[s] + static_cast<int64_t>(tok) * a.topk;
  const int64_t* base = a.tile_base + static_cast<int64_t>(s) * a.buckets * a.tiles;
  for (int k = 0; k < a.topk; ++k) {
    const int e = ids[k];
    if (e < 0 || e >= E) continue;
    const int d = e / epr;
    const int b = a.dedup ? d : e;
    const int64_t off = base[static_cast<int64_t>(b) * a.tiles + tile] - sdispl[d];
    pos[k] = static_cast<int32_t>(rdispl[d] + off + pos[k]);
  }
}

int launch_moe_route(const MoeRouteArgs& a, cudaStream_t s) {
  const unsigned grid = static_cast<unsigned>(a.n * a.tiles);
  const size_t smem = static_cast<size_t>(a.buckets) * kWords * sizeof(uint32_t);
  static int smem_set[COLL_MAX_RANKS] = {0};  // per device ordinal: largest limit set so far
  const int ok = allow_dynamic_smem(reinterpret_cast<const void*>(k_moe_count), smem, smem_set);
  if (ok != COLL_OK) return ok;
  launch_pdl(k_moe_count, dim3(grid), dim3(kTile), smem, s, a);  // tokens == 0 still zeroes the counts
  int st = launch_status(cudaGetLastError());
  if (st != COLL_OK) return st;
  launch_pdl(k_moe_scan, dim3(a.n), dim3(kScanThreads), 0, s, a);
  st = launch_status(cudaGetLastError());
  if (st != COLL_OK) return st;
  launch_pdl(k_moe_pos, dim3(std::max(grid, 1u)), dim3(kTile), 0, s, a);
  return launch_status(cudaGetLastError());
}

// --------------------------------------------------------------- dispatch ----

struct RowTargets {
  char* dst[kMaxTopk];
};

template <int U>
__global__ void __launch_bounds__(kMoveThreads) k_moe_dispatch(const __grid_constant__ MoeMoveArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ char* cand[kMaxTopk];
  __shared__ char* dst[kMaxTopk];  // cand with repeats of an earlier choice's row dropped
  __shared__ int nbad;
  const int64_t rows = static_cast<int64_t>(a.n) * a.tokens;
  const uint64_t ru = a.row_bytes / U;
  int bad = 0;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const int s = static_cast<int>(row / a.tokens);
    const int t = static_cast<int>(row % a.tokens);
    if (threadIdx.x < a.topk) {
      const int64_t j = static_cast<int64_t>(t) * a.topk + threadIdx.x;
      const int e = a.ids[s][j];
      const int64_t p = a.pos[s][j];
      const int d = e / a.epr;
      if (e < 0 || d >= a.n || p < 0 || p >= a.capacity) {
        cand[threadIdx.x] = nullptr;
        ++bad;
      } else {
        cand[threadIdx.x] = a.y[d] + static_cast<uint64_t>(p) * a.row_bytes;
      }
    }
    __syncthreads();
    if (threadIdx.x < a.topk) {
      char* c = cand[threadIdx.x];
      for (int k2 = 0; k2 < threadIdx.x; ++k2)
        if (cand[k2] == c) c = nullptr;
      dst[threadIdx.x] = c;
    }
    __syncthreads();
    const char* src = a.x[s] + static_cast<uint64_t>(t) * a.row_bytes;
    for (uint64_t u = threadIdx.x; u < ru; u += blockDim.x) {
      const auto v = ldu<U>(src + u * U);
      for (int k = 0; k < a.topk; ++k) {
        char* d = dst[k];
        if (d != nullptr) stu<U>(d + u * U, v);
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) nbad = 0;
  __syncthreads();
  if (bad) atomicAdd(&nbad, bad);
  __syncthreads();
  if (threadIdx.x == 0) report(a.status, COLL_DEV_SPLIT_OVERFLOW, nbad);
}

// Bulk-copy dispatch: one warp per CTA.  Each token row is loaded once into
// a shared-memory stage with cp.async.bulk and written to its topk receive
// rows with bulk stores; when a row's load is issued, lanes 0..topk-1 also
// look up where it goes, so the stores never wait on those lookups.
constexpr int kDispStages = 4;
constexpr uint32_t kDispMaxRow = 32768;  // bytes of one row in a stage

__global__ void __launch_bounds__(32) k_moe_dispatch_tma(const __grid_constant__ MoeMoveArgs a, uint32_t stage_bytes) {
  extern __shared__ __align__(128) unsigned char stage_buf[];
  __shared__ __align__(8) uint64_t bar[kDispStages];
  __shared__ char* dst[kDispStages][kMaxTopk];
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x;
  const uint32_t rb = static_cast<uint32_t>(a.row_bytes);
  if (lane == 0) {
    for (int st = 0; st < kDispStages; ++st) mbar_init(&bar[st], 1);
    fence_barrier_init();
  }
  __syncwarp();
  const uint64_t rows = static_cast<uint64_t>(a.n) * a.tokens;
  const uint64_t stride = gridDim.x;
  int bad = 0;
  auto issue = [&](uint64_t row, int st) {
    const int s = static_cast<int>(row / a.tokens);
    const int t = static_cast<int>(row % a.tokens);
    if (lane < a.topk) {
      const int64_t j = static_cast<int64_t>(t) * a.topk + lane;
      const int e = a.ids[s][j];
      const int64_t p = a.pos[s][j];
      const int d = e / a.epr;
      if (e < 0 || d >= a.n || p < 0 || p >= a.capacity) {
        dst[st][lane] = nullptr;
        ++bad;
      } else {
        dst[st][lane] = a.y[d] + static_cast<uint64_t>(p) * rb;
      }
    }
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar[st], rb);
      bulk_load(stage_buf + st * stage_bytes, a.x[s] + static_cast<uint64_t>(t) * rb, rb, &bar[st]);
    }
  };
  int inflight = 0;
  for (int st = 0; st < kDispStages && blockIdx.x + st * stride < rows; ++st, ++inflight) issue(blockIdx.x + st * stride, st);
  __syncwarp();
  int i = 0;
  for (uint64_t row = blockIdx.x; row < rows; row += stride, ++i) {
    const int st = i % kDispStages;
    int ok = 1;
    if (lane == 0) {
      ok = mbar_wait_bounded(&bar[st], (i / kDispStages) & 1) ? 1 : 0;
      if (ok) {
        for (int k = 0; k < a.topk; ++k) {
          char* d = dst[st][k];
          for (int k2 = 0; k2 < k && d != nullptr; ++k2)
            if (dst[st][k2] == d) d = nullptr;  // the same row as an earlier choice: written once
          if (d != nullptr) bulk_store(d, stage_buf + st * stage_bytes, rb);
        }
        bulk_commit();
      }
    }
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (!ok) {
      if (lane == 0) {
        report(a.status, COLL_DEV_TIMEOUT, 1);
        bulk_wait_all();
        for (int k = 1; k < inflight; ++k)
          mbar_wait_bounded(&bar[(i + k) % kDispStages], ((i + k) / kDispStages) & 1);
      }
      return;
    }
    --inflight;
    const uint64_t nxt = row + kDispStages * stride;
    if (nxt < rows) {
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();  // the stage and its destination list are free again
      issue(nxt, st);
      ++inflight;
      __syncwarp();
    }
  }
  if (lane == 0) bulk_wait_all();
  report_warp(a.status, COLL_DEV_SPLIT_OVERFLOW, bad);
}

static int pick_unit(uint64_t bits) {
  if ((bits & 15) == 0) return 16;
  if ((bits & 7) == 0) return 8;
  if ((bits & 3) == 0) return 4;
  if ((bits & 1) == 0) return 2;
  return 1;
}

static unsigned move_grid(int64_t rows) {
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  return static_cast<unsigned>(std::max<int64_t>(1, std::min(rows, cap)));
}

int launch_moe_dispatch(const MoeMoveArgs& a, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(a.n) * a.tokens;
  if (rows == 0 || a.row_bytes == 0) return COLL_OK;
  uint64_t bits = a.row_bytes;
  for (int r = 0; r < a.n; ++r) bits |= reinterpret_cast<uintptr_t>(a.x[r]) | reinterpret_cast<uintptr_t>(a.y[r]);
  // whole rows through shared memory once there are enough of them
  const uint32_t stage_bytes = static_cast<uint32_t>((a.row_bytes + 127) / 128 * 128);
  const int64_t per_sm = std::max<int64_t>(1, (200 * 1024) / (kDispStages * static_cast<int64_t>(stage_bytes)));
  const int64_t resident = static_cast<int64_t>(num_sms()) * per_sm;
  if ((bits & 15) == 0 && a.row_bytes <= kDispMaxRow && rows >= 4 * resident) {
    const size_t smem = static_cast<size_t>(kDispStages) * stage_bytes;
    static int smem_set[COLL_MAX_RANKS] = {0};  // per device ordinal: largest limit set so far
    const int ok = allow_dynamic_smem(reinterpret_cast<const void*>(k_moe_dispatch_tma), smem, smem_set);
    if (ok != COLL_OK) return ok;
    // one CTA per kDispStages rows, launched in order: measured faster than a
    // resident grid walking the rows (8 x 4096 rows of 14 KB: 662 against 751 us)
    const uint64_t grid = stream_grid(static_cast<uint64_t>(rows), kDispStages);
    launch_pdl(k_moe_dispatch_tma, dim3(static_cast<unsigned>(grid)), dim3(32), smem, s, a,
               stage_bytes);
    return launch_status(cudaGetLastError());
  }
  const unsigned grid = move_grid(rows);
  switch (pick_unit(bits)) {
    case 16: launch_pdl(k_moe_dispatch<16>, dim3(grid), dim3(kMoveThreads), 0, s, a); break;
    case 8: launch_pdl(k_moe_dispatch<8>, dim3(grid), dim3(kMoveThreads), 0, s, a); break;
    case 4: launch_pdl(k_moe_dispatch<4>, dim3(grid), dim3(kMoveThreads), 0, s, a); break;
    case 2: launch_pdl(k_moe_dispatch<2>, dim3(grid), dim3(kMoveThreads), 0, s, a); break;
    default: launch_pdl(k_moe_dispatch<1>, dim3(grid), dim3(kMoveThreads), 0, s, a); break;
  }
  return launch_status(cudaGetLastError());
}

// ---------------------------------------------------------------- combine ----

template <int DT, bool VEC, int TK>  // TK: top-k known at compile time (0 = runtime)
__global__ void __launch_bounds__(kMoveThreads) k_moe_combine(const __grid_constant__ MoeMoveArgs a) {
  pdl_wait();
  pdl_trigger();
  using S = typename Elem<DT>::S;
  constexpr int VN = Vec<DT>::kN;
  constexpr int ES = Elem<DT>::kSize;
  __shared__ const char* src[kMaxTopk];
  __shared__ float wk[kMaxTopk];
  __shared__ int nbad;
  const int topk = TK > 0 ? TK : a.topk;
  const int64_t rows = static_cast<int64_t>(a.n) * a.tokens;
  const uint64_t relems = a.row_bytes / ES;
  int bad = 0;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const int s = static_cast<int>(row / a.tokens);
    const int t = static_cast<int>(row % a.tokens);
    if (threadIdx.x < topk) {
      const int64_t j = static_cast<int64_t>(t) * topk + threadIdx.x;
      const int e = a.ids[s][j];
      const int64_t p = a.pos[s][j];
      const int d = e / a.epr;
      wk[threadIdx.x] = a.w[s][j];
      if (e < 0 || d >= a.n || p < 0 || p >= a.capacity) {
        src[threadIdx.x] = nullptr;
        ++bad;
      } else {
        src[threadIdx.x] = a.x[d] + static_cast<uint64_t>(p) * a.row_bytes;
      }
    }
    __syncthreads();
    char* out = a.y[s] + static_cast<uint64_t>(t) * a.row_bytes;
    if constexpr (VEC && TK > 0) {
      const char* sp[TK];
      float w[TK];
#pragma unroll
      for (int k = 0; k < TK; ++k) {
        sp[k] = src[k];
        w[k] = wk[k];
      }
      const uint64_t units = relems / VN;
      auto one = [&](const uint4 (&x)[TK], uint64_t u) {
        Vec<DT> acc;
#pragma unroll
        for (int k = 0; k < TK; ++k) {
          Vec<DT> v;
          widen16<DT>(x[k], v);
#pragma unroll
          for (int i = 0; i < VN; ++i) {
            const float prod = __fmul_rn(w[k], v.v[i]);
            acc.v[i] = k == 0 ? prod : __fadd_rn(acc.v[i], prod);
          }
        }
        st16(out + u * 16, narrow16<DT>(acc));
      };
      uint64_t u = threadIdx.x;
      for (; u + blockDim.x < units; u += 2 * blockDim.x) {  // two units per pass: 2 x TK loads in flight
        uint4 x0[TK], x1[TK];
#pragma unroll
        for (int k = 0; k < TK; ++k) {
          x0[k] = sp[k] != nullptr ? ld16(sp[k] + u * 16) : make_uint4(0, 0, 0, 0);
          x1[k] = sp[k] != nullptr ? ld16(sp[k] + (u + blockDim.x) * 16) : make_uint4(0, 0, 0, 0);
        }
        one(x0, u);
        one(x1, u + blockDim.x);
      }
      if (u < units) {
        uint4 x0[TK];
#pragma unroll
        for (int k = 0; k < TK; ++k) x0[k] = sp[k] != nullptr ? ld16(sp[k] + u * 16) : make_uint4(0, 0, 0, 0);
        one(x0, u);
      }
    } else if constexpr (VEC) {
      for (uint64_t u = threadIdx.x; u < relems / VN; u += blockDim.x) {
        Vec<DT> acc;
        for (int k = 0; k < topk; ++k) {
          Vec<DT> v;
          if (src[k] != nullptr) widen16<DT>(ld16(src[k] + u * 16), v);
          else widen16<DT>(make_uint4(0, 0, 0, 0), v);
          const float w = wk[k];
#pragma unroll
          for (int i = 0; i < VN; ++i) {
            const float prod = __fmul_rn(w, v.v[i]);
            acc.v[i] = k == 0 ? prod : __fadd_rn(acc.v[i], prod);
          }
        }
        st16(out + u * 16, narrow16<DT>(acc));
      }
    } else {
      for (uint64_t e = threadIdx.x; e < relems; e += blockDim.x) {
        float acc = 0.f;
        for (int k = 0; k < topk; ++k) {
          const float v = src[k] != nullptr ? widen1<DT>(*reinterpret_cast<const S*>(src[k] + e * ES)) : 0.f;
          const float prod = __fmul_rn(wk[k], v);
          acc = k == 0 ? prod : __fadd_rn(acc, prod);
        }
        *reinterpret_cast<S*>(out + e * ES) = narrow1<DT>(acc);
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) nbad = 0;
  __syncthreads();
  if (bad) atomicAdd(&nbad, bad);
  __syncthreads();
  if (threadIdx.x == 0) report(a.status, COLL_DEV_SPLIT_OVERFLOW, nbad);
}

template <int DT>
static int launch_combine_dt(const MoeMoveArgs& a, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(a.n) * a.tokens;
  uint64_t bits = a.row_bytes;
  for (int r = 0; r < a.n; ++r) bits |= reinterpret_cast<uintptr_t>(a.x[r]) | reinterpret_cast<uintptr_t>(a.y[r]);
  void (*fn)(MoeMoveArgs) = (bits & 15) == 0 && a.topk == 8 ? k_moe_combine<DT, true, 8>
                            : (bits & 15) == 0                ? k_moe_combine<DT, true, 0>
                                                              : k_moe_combine<DT, false, 0>;
  // a CTA per token row, launched in order
  const unsigned grid = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(rows, kMaxStreamGrid)));
  launch_pdl(fn, dim3(grid), dim3(kMoveThreads), 0, s, a);
  return launch_status(cudaGetLastError());
}

int launch_moe_combine(const MoeMoveArgs& a, coll_dtype_t dt, cudaStream_t s) {
  if (static_cast<int64_t>(a.n) * a.tokens == 0 || a.row_bytes == 0) return COLL_OK;
  switch (dt) {
    case COLL_BF16: return launch_combine_dt<COLL_BF16>(a, s);
    case COLL_FP16: return launch_combine_dt<COLL_FP16>(a, s);
    case COLL_FP32: return launch_combine_dt<COLL_FP32>(a, s);
    default: return COLL_ERR_UNSUPPORTED;
  }
}

}  // namespace mvr
