// Host-side interface between the C-ABI layer (api.cu) and the kernel files.
// Argument structs are passed to kernels by value as __grid_constant__
// parameters (sm_100a accepts up to 32 KB of kernel parameters).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "coll.h"

namespace mvr {

constexpr int kMaxRanksH = COLL_MAX_RANKS;
constexpr int kBlockThreads = 256;  // threads per CTA of the element-wise kernels

int num_sms();                      // SM count of the current device (cached)
int resident_ctas(const void* fn, int threads, size_t smem);  // CTAs of fn that fit at once on the device
constexpr uint64_t kMaxStreamGrid = 1ull << 30;  // CTAs of one streaming launch at most
uint64_t stream_grid(uint64_t units, int threads);  // one work item per thread, at most kMaxStreamGrid CTAs
int elem_size(coll_dtype_t dt);     // 2 or 4, 0 for an unknown dtype
int launch_status(cudaError_t e);   // COLL_OK or COLL_ERR_CUDA (remembers the error text)
// Raise `fn`'s dynamic shared memory limit to at least `bytes` on the current
// device (`done` holds one entry per device ordinal, the largest limit set so
// far).  Called before every launch that uses dynamic shared memory, whatever
// its size: the 48 KB default counts the kernel's static shared memory too.
int allow_dynamic_smem(const void* fn, size_t bytes, int* done);

// ----------------------------------------------------------- reductions ----
struct ReduceArgs {
  const char* in[kMaxRanksH];
  char* out[kMaxRanksH];
  uint64_t count;   // elements of the reduced index range of every input
  uint64_t seg;     // elements per slice (owner segment / output block); ignored by ONESHOT
  int nin;          // ranks reduced
  int nout;         // M_ALL: output ranks written
  int nslices;      // slices interleaved over blockIdx.x
};
// mode: mvr::ReduceMode.  vec: all addresses and slice starts 16-byte aligned.
int launch_reduce(const ReduceArgs& a, coll_dtype_t dt, coll_op_t op, int mode, bool vec,
                  int blocks_per_slice, cudaStream_t s);

struct RingStepArgs {
  const char* in[kMaxRanksH];
  char* out[kMaxRanksH];
  char* partial;    // arithmetic-type partials, indexed by element
  uint64_t count, seg;
  int n, k;         // ranks, step 1 .. n-1 of the reduce-scatter phase
};
int launch_ring_rs_step(const RingStepArgs& a, coll_dtype_t dt, coll_op_t op, bool vec,
                        cudaStream_t s);
// The whole stream-ordered ring (RING_STEPS): N-1 reduce-scatter step
// launches whose partials live at `partial` (count elements of the
// arithmetic type), then N-1 all-gather copy launches.  Shared by
// coll_all_reduce and coll_all_reduce_ring_noalloc, so both give the same bits.
int launch_ring_steps(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                      char* partial, bool vec, cudaStream_t s);

size_t twoshot_ll_workspace(int n, size_t count, int es);
int launch_twoshot_ll(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                      void* workspace, int* status, cudaStream_t s);
size_t twoshot_ll128_workspace(int n, size_t count, int es);
int launch_twoshot_ll128(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt,
                         coll_op_t op, void* workspace, int* status, cudaStream_t s);
size_t ring_ll_workspace(int n, size_t count, int es);
int launch_ring_ll(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                   void* workspace, int* status, cudaStream_t s);
bool ring_cluster_supported(int n);
int launch_ring_cluster(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                        int* status, cudaStream_t s);
bool ring_cta_supported(int n);
bool ring_lane_supported(int n);
int launch_ring_lane(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                     cudaStream_t s);
int launch_ring_cta(const char* const* in, char* const* out, int n, size_t count, coll_dtype_t dt, coll_op_t op,
                    bool wire, cudaStream_t s);
int launch_wait_flag(const uint32_t* flag, uint32_t expect, uint32_t budget_us, int* status, cudaStream_t s);

// ---------------------------------------------------------------- copies ----
struct FanoutArgs {
  const char* src[kMaxRanksH];
  char* dst[kMaxRanksH];
  uint64_t bytes;       // bytes per source
  uint64_t dst_stride;  // dst for (source r, destination q) = dst[q] + r * dst_stride
  int ns, nd;
  int skip_diag;        // skip q == r (in-place all-gather)
  int* status;          // optional device status pair (bounded-wait timeouts)
};
int launch_fanout(const FanoutArgs& a, cudaStream_t s);

struct CopyJob {
  const char* src;
  char* dst;
  uint64_t bytes;
};
// any number of independent 1-D copies (split over several launches if needed)
int launch_copy_jobs(const CopyJob* jobs, int njobs, cudaStream_t s);

struct GatherRowsArgs {
  const char* src[kMaxRanksH];
  char* dst;
  uint64_t rows, row_bytes, dst_pitch;
  int n;
};
int launch_gather_rows(const GatherRowsArgs& a, cudaStream_t s);

// --------------------------------------------------------------- packets ----
// One codec launch encodes (pack) or decodes (unpack) the equally long
// messages of n virtual ranks, blockIdx.y selecting the rank.
struct CodecArgs {
  const uint8_t* in[kMaxRanksH];  // messages (pack) or packets (unpack)
  uint8_t* out[kMaxRanksH];       // packets (pack) or messages (unpack)
  uint64_t bytes;                 // message bytes per rank
  uint64_t step;                  // the flag
  int n;
  int* status;                    // unpack: flag mismatches (may be null)
};
int launch_ll_pack(const CodecArgs& a, int proto, cudaStream_t s);
int launch_ll_unpack(const CodecArgs& a, int proto, cudaStream_t s);

struct PackedReduceArgs {
  const char* in[kMaxRanksH];
  char* out[kMaxRanksH];
  uint64_t nlines;       // lines per rank
  uint64_t payload_bytes;
  uint64_t step;
  int n;
  int* status;
};
int launch_all_reduce_packed(const PackedReduceArgs& a, coll_dtype_t dt, coll_op_t op, int proto,
                             cudaStream_t s);

// -------------------------------------------------------------------- MoE ----
struct MoeRouteArgs {
  const int32_t* ids[kMaxRanksH];
  int32_t* pos[kMaxRanksH];
  int64_t* send_counts;  // [N*N]
  int64_t* send_displs;  // [N*N]
  int64_t* recv_displs;  // [N*N] (d-major)
  int32_t* tile_cnt;     // workspace [N][E][tiles]
  int64_t* tile_base;    // workspace [N][E][tiles]
  int* status;
  int n, tokens, topk, n_experts, tiles;
  // route buckets: experts (one row per (token, expert)), or destination
  // ranks when deduplicated (one row per (token, rank)); bpr = buckets per rank
  int dedup, buckets, bpr;
};
size_t moe_route_workspace(int n, int tokens, int topk, int n_experts);
int launch_moe_route(const MoeRouteArgs& a, cudaStream_t s);

struct MoeMoveArgs {
  const char* x[kMaxRanksH];      // dispatch: token rows; combine: expert outputs y
  char* y[kMaxRanksH];            // dispatch: receive buffers; combine: outputs
  const int32_t* ids[kMaxRanksH];
  const int32_t* pos[kMaxRanksH];
  const float* w[kMaxRanksH];
  uint64_t row_bytes;
  int64_t capacity;
  int* status;
  int n, tokens, topk, epr;
};
int launch_moe_dispatch(const MoeMoveArgs& a, cudaStream_t s);
int launch_moe_combine(const MoeMoveArgs& a, coll_dtype_t dt, cudaStream_t s);

}  // namespace mvr
