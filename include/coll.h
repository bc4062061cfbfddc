/*
 * coll.h -- C ABI of the virtual-rank collectives engine (libmvrcoll.so).
 *
 * One B200 holds N "virtual ranks": N disjoint buffers in its own HBM.  Every
 * entry point below performs the data movement (and reduction) of one
 * collective over those buffers with hand-written sm_100a kernels.  Nothing
 * crosses GPUs.
 *
 * Sources (cited by page title and section):
 *   [TUT]  vLLM collectives tutorial, gsyq.cn/news/307221 -- sections
 *          1 Broadcast ... 8 All-to-All.
 *   [RLL]  "From NCCL Ring LL to PCIe IPC AllReduce" (hjcheng0602.cn) --
 *          sections "Traditional LL Protocols" and "Pro5000 ?".
 *   [TPC]  TP communication-overhead essay, 52jiny.com thread-1337 -- the
 *          section on how communication erodes scaling (ring steps).
 *   [A2A]  sglang PR 27492 summary (prhub) -- GroupCoordinator
 *          all_to_all_single, "implementation breakdown".
 *   [BCS]  sglang PR 33307 summary (prhub) -- single-image broadcast.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointer arrays (`const void* const* send`, ...) are HOST arrays of N
 *   DEVICE pointers, one per virtual rank, read during the call only.  All
 *   device buffers belong to the caller and must stay alive until the work
 *   enqueued on `stream` has finished.  The library never allocates device
 *   memory at run time; kernels that need scratch take a caller-provided
 *   `workspace` whose size the matching *_workspace_size() function returns.
 *   The one exception is coll_all_reduce_ring_noalloc (near the end of this
 *   file), whose scratch is a fixed array compiled into the library.
 * - Every call only ENQUEUES work on `stream` (NULL = legacy default
 *   stream) and never synchronises.  Calls are thread-safe; the library keeps
 *   no state besides per-device caches (the SM count, kernel attributes set
 *   once, and the address of the no-allocation entry point's array).
 * - Counts are in ELEMENTS of `dtype` unless stated otherwise; buffers are
 *   dense (contiguous).  N = nranks, 1 <= N <= COLL_MAX_RANKS.
 * - Return value: COLL_OK or a negative COLL_ERR_* code, decided on the host
 *   before anything is enqueued (argument errors) or right after the launch
 *   (COLL_ERR_CUDA).  coll_strerror() gives a message.
 * - Errors only the device can see (a packet flag that does not match, a
 *   row index beyond a receive buffer, a malformed route, a used-up LL call
 *   counter) are reported in an
 *   optional device word pair `int d_status[2]`: d_status[0] receives the
 *   first COLL_DEV_* code raised (atomic compare-and-swap from 0) and
 *   d_status[1] is incremented by the number of offending items.  The caller
 *   zeroes it.  Kernels never trap and never wait on a flag.
 * - count == 0 is a successful no-op.  N == 1 is a copy (or nothing when
 *   in place), as world size 1 is in [A2A] "implementation breakdown", item 3.
 * - 16-byte aligned buffers take the vectorised path; anything else falls
 *   back to an element-wise path with the same result.
 * - Overlap between buffers is an error (COLL_ERR_ALIAS) except the in-place
 *   forms each function names.
 *
 * Arithmetic (reductions): inputs are widened exactly to fp32 (int32 stays
 * int32), combined in rank order 0, 1, ..., N-1 with IEEE binary32
 * round-to-nearest-even operations (no fused multiply-add), and rounded once
 * to the storage type (round to nearest, ties to even; a NaN result becomes
 * the canonical NaN 0x7FC0 for bf16, 0x7E00 for fp16, 0x7FC00000 for fp32).  MAX/MIN keep the earlier rank on ties
 * and propagate NaN.  int32 SUM/PROD wrap modulo 2^32.  The ring all-reduce
 * is the one exception to the rank order (see coll_all_reduce).
 */
#ifndef MVR_COLL_H
#define MVR_COLL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define COLL_API __attribute__((visibility("default")))
#else
#define COLL_API
#endif

typedef struct CUstream_st* coll_stream_t; /* identical to cudaStream_t */

typedef enum { COLL_BF16 = 0, COLL_FP16 = 1, COLL_FP32 = 2, COLL_INT32 = 3 } coll_dtype_t;
typedef enum { COLL_SUM = 0, COLL_MAX = 1, COLL_MIN = 2, COLL_PROD = 3 } coll_op_t;
typedef enum {
  COLL_ALGO_AUTO = 0,    /* the measured fastest: ONESHOT or TWOSHOT by ranks and size */
  COLL_ALGO_ONESHOT = 1, /* every rank reads all N inputs itself            */
  COLL_ALGO_TWOSHOT = 2, /* owner s reduces segment s, sends it to everyone */
  COLL_ALGO_RING = 3,    /* 2(N-1) neighbour steps: RING_LANE / RING_CTA, else RING_STEPS */
  COLL_ALGO_RING_LL = 4, /* the same ring in one launch, LL packets between ranks */
  COLL_ALGO_RING_CLUSTER = 5, /* the same ring, ranks = CTAs of a cluster, hops over DSMEM */
  COLL_ALGO_RING_STEPS = 6,   /* the same ring, one stream-ordered launch per step */
  COLL_ALGO_TWOSHOT_LL = 7,   /* TWOSHOT in one launch, LL packets between ranks */
  COLL_ALGO_RING_CTA = 8,     /* the same ring, ranks = warp groups of one CTA, hops in shared memory */
  COLL_ALGO_TWOSHOT_LL128 = 9, /* TWOSHOT in one launch, LL128 packets between ranks */
  COLL_ALGO_RING_LANE = 10,    /* the same ring, ranks = lanes of one warp, hops by warp shuffles */
  COLL_ALGO_RING_WIRE = 11     /* the ring's order, partials rounded to the buffer type at every hop */
} coll_algo_t;
typedef enum { COLL_PROTO_SIMPLE = 0, COLL_PROTO_LL = 1, COLL_PROTO_LL128 = 2 } coll_proto_t;

#define COLL_MAX_RANKS 64
#define COLL_MAX_EXPERTS 1024

/* synchronous return codes */
#define COLL_OK 0
#define COLL_ERR_INVALID_ARG (-1) /* null pointer, rank out of range, bad size, step 0 */
#define COLL_ERR_UNSUPPORTED (-2) /* dtype / op / algo combination not provided      */
#define COLL_ERR_ALIAS (-3)       /* buffers overlap in a way the op does not allow  */
#define COLL_ERR_CUDA (-4)        /* a launch failed                                 */
#define COLL_ERR_WORKSPACE (-5)   /* workspace missing, too small or misaligned      */

/* device status codes (d_status[0]) */
#define COLL_DEV_OK 0
#define COLL_DEV_FLAG_MISMATCH 1  /* a packet line's flag differed from `step`         */
#define COLL_DEV_TIMEOUT 2        /* reserved for bounded in-kernel waits              */
#define COLL_DEV_SPLIT_OVERFLOW 3 /* a row index fell outside the receive buffer       */
#define COLL_DEV_BAD_ROUTE 4      /* expert id out of range, or repeated within a token */
#define COLL_DEV_EPOCH_WRAP 5     /* an LL workspace's call counter is used up: the call did
                                     nothing; zero-fill the workspace before the next call */

/* Calls one zero-filled workspace serves in RING_LL and TWOSHOT_LL (the call
 * counter is the little-endian u32 at byte 0 of the workspace). */
#define COLL_RING_LL_CALLS_PER_FILL (1u << 25)
#define COLL_TWOSHOT_LL_CALLS_PER_FILL (1u << 30)

/* ------------------------------------------------------------------------ */

/* Broadcast ([TUT] 1.1; [BCS] "key code"): after the call every rank's
 * buffer holds the bytes of bufs[src].  bufs[src] is only read, the others
 * only written; all N buffers are `count` elements and must not overlap.
 * The copy is bit-exact and dtype-agnostic (dtype only fixes the element
 * size). */
COLL_API int coll_broadcast(void* const* bufs, int nranks, size_t count, coll_dtype_t dtype, int src,
                   coll_stream_t stream);

/* Gather ([TUT] 2.1, 2.2.1): rank `dst` receives every rank's block in rank
 * order; other ranks receive nothing.  Each send[r] is a dense
 * [rows, cols_per_rank] block; recv_dst is [rows, N * cols_per_rank] and
 * recv_dst[row][r * cols_per_rank + j] = send[r][row][j] (blocks joined along
 * the last dimension, the vocab-sharded logits picture of 2.2.1).  rows == 1
 * is the flat concatenation.  In place: send[dst] may already be block dst
 * of recv_dst when rows == 1. */
COLL_API int coll_gather(const void* const* send, void* recv_dst, int nranks, size_t rows,
                size_t cols_per_rank, coll_dtype_t dtype, int dst, coll_stream_t stream);

/* Reduce ([TUT] 3.1): recv_dst[i] = op over r = 0..N-1 of send[r][i], for
 * rank `dst` only.  In place: recv_dst == send[dst]. */
COLL_API int coll_reduce(const void* const* send, void* recv_dst, int nranks, size_t count,
                coll_dtype_t dtype, coll_op_t op, int dst, coll_stream_t stream);

/* Scatter ([TUT] 4.1): send_src holds N * count_per_rank elements cut into
 * N equal blocks; recv[r] receives block r.  In place: recv[src] may be
 * block src of send_src. */
COLL_API int coll_scatter(const void* send_src, void* const* recv, int nranks, size_t count_per_rank,
                 coll_dtype_t dtype, int src, coll_stream_t stream);

/* ReduceScatter ([TUT] 5.1, 5.3): every send[q] holds N * recv_count
 * elements; recv[r][i] = op over q of send[q][r * recv_count + i] (rank r
 * keeps block r of the reduction).  In place: recv[r] may be block r of
 * send[r]. */
COLL_API int coll_reduce_scatter(const void* const* send, void* const* recv, int nranks,
                        size_t recv_count, coll_dtype_t dtype, coll_op_t op,
                        coll_stream_t stream);

/* AllReduce ([TUT] 6.1): every recv[q][i] = op over r of send[r][i].
 *  ONESHOT ([RLL] "Pro5000 ?", the one-shot scheme it compares with): each
 *    output rank reads all N inputs and reduces them itself; not in place.
 *  TWOSHOT ([RLL] "Pro5000 ?", the A/B/C/D example): the element range is cut
 *    into N owner segments of ceil(count/N) elements rounded up to 16 bytes
 *    (the last ones may be short or empty); owner s reduces segment s across
 *    all ranks and writes it to every rank.  One fused kernel.
 *  RING ([TPC]; NCCL's ring kernel named in [RLL]): 2(N-1) steps on the
 *    ring r -> r+1 over the same N chunks: chunk c starts on rank c+1, every
 *    step moves it one rank on where that rank adds its own values (so chunk
 *    c is accumulated in the order c+1, ..., N-1, 0, ..., c), and the N-1
 *    all-gather steps pass the finished chunks round.  Partials travel in
 *    fp32 (int32 for int32); the result may differ from the rank-order
 *    reduction by rounding only.  When 2 <= N <= 8 and every buffer is
 *    16-byte aligned it runs in one launch, as the form measured fastest on
 *    B200: RING_LANE for N == 2, for N <= 4 up to 256 KiB and for N >= 5 up
 *    to 16 KiB per rank, RING_CTA above; otherwise as RING_STEPS.  Every
 *    form gives the same result bit for bit.
 *    coll_all_reduce_form() tells which.  `workspace`:
 *    coll_all_reduce_workspace_size() bytes, 16-byte aligned: a 256-byte
 *    header whose bytes 16..23 receive the status pair of the one-launch
 *    form (int[2], cleared by the caller; COLL_DEV_TIMEOUT if a bounded wait
 *    ran out), then the partials of the stream-ordered form.
 *  RING_STEPS: the RING schedule as 2(N-1) stream-ordered launches, one per
 *    step (the launch boundary is the step's synchronisation); partials in
 *    the workspace after its header.  Nothing waits, so it cannot time out.
 *  RING_LL ([RLL] "Traditional LL Protocols", "Pro5000 ?": NCCL's Ring LL
 *    kernel): the RING schedule, chunk order and rounding (bit-identical
 *    result) in ONE cooperative launch.  Virtual rank r is a set of CTAs; it
 *    sends each step's values to rank r+1 as LL lines [4 B value | 4 B flag]
 *    in a FIFO in `workspace`, and rank r+1 re-reads each 16-byte group until
 *    both flags match before using it.  Waits are bounded (about 1 s); a wait
 *    that runs out makes every CTA stop and raises COLL_DEV_TIMEOUT in the
 *    status pair at byte offset 16 of the workspace (int[2], cleared by the
 *    caller).  The workspace (coll_all_reduce_workspace_size() bytes,
 *    256-byte aligned) must be zero-filled once before its first use and
 *    serves one call at a time; the library keeps a call counter in it.
 *    The counter occupies the flag's upper 25 bits, so one fill serves
 *    COLL_RING_LL_CALLS_PER_FILL calls: a call made after those (its flags
 *    would repeat those of the first call, and a line left unwritten that
 *    long would pass for current) enqueues a kernel that does nothing but
 *    raise COLL_DEV_EPOCH_WRAP in the status pair; zero-fill the workspace
 *    again to go on.
 *    Buffers that are not 16-byte aligned take the RING_STEPS path.
 *  RING_CLUSTER: the RING schedule, chunk order and rounding (bit-identical
 *    result) in one launch of thread-block clusters of N CTAs, CTA r playing
 *    virtual rank r: each hop is an asynchronous store into the next CTA's
 *    shared memory over the SM-to-SM network that completes that CTA's
 *    mbarrier, so the partials never touch HBM.  The clusters are about as
 *    many as fit on the GPU at once and walk the message tile by tile.
 *    Needs 2 <= N <= 8 and 16-byte aligned buffers; otherwise, if a
 *    RING-sized `workspace` is given, the call takes the RING_STEPS path,
 *    else it returns COLL_ERR_UNSUPPORTED.  `workspace` is optional:
 *    when at least 24 bytes are given, bytes 16..23 receive the status pair
 *    (COLL_DEV_TIMEOUT if a bounded wait ran out).
 *  RING_CTA: the RING schedule, chunk order and rounding (bit-identical
 *    result) in one launch in which every CTA holds all N virtual ranks,
 *    one warp each: each hop is a store into a shared-memory slot of the
 *    same SM and one CTA-wide barrier, so the partials never leave the SM
 *    and nothing waits on another CTA.  The grid has one CTA per tile of
 *    the message, launched in order.  Needs 2 <= N <= 8 and 16-byte aligned
 *    buffers, with the same fallback as RING_CLUSTER; `workspace` is
 *    optional and unused (this form raises no device status).
 *  RING_LANE: the RING schedule, chunk order and rounding (bit-identical
 *    result) in one launch in which the N virtual ranks are N lanes of one
 *    warp (a warp holds 32 / W such rings, W = N rounded up to a power of
 *    two, each on its own 16-byte column of every chunk): each hop is a
 *    warp shuffle from lane r to lane r+1, so the partials stay in
 *    registers, no shared memory or barrier is used, and HBM sees each
 *    input and output byte once.  Needs 2 <= N <= 8 and 16-byte aligned
 *    buffers, with the same fallback as RING_CLUSTER; `workspace` is
 *    optional and unused (this form raises no device status).
 *  RING_WIRE: the RING schedule and chunk order with a different result:
 *    every reduce-scatter hop carries the partial rounded to the buffers'
 *    type (a ring whose messages carry the buffer dtype), so each receiver
 *    widens it, combines its own values in fp32 and rounds again.  For bf16
 *    / fp16 SUM and PROD the result differs from RING's by those extra
 *    roundings (no bound is promised); for fp32, int32, MAX and MIN it is
 *    RING's bit for bit.  Runs as RING_CTA with half the hop bytes for
 *    bf16 / fp16; needs 2 <= N <= 8 and 16-byte aligned buffers
 *    (COLL_ERR_UNSUPPORTED otherwise: there is no stream-ordered form);
 *    `workspace` is ignored.
 *  TWOSHOT_LL ([RLL] "Traditional LL Protocols" and the "Pro5000 ?" two-shot,
 *    fused): the TWOSHOT segments and arithmetic (bit-identical result) in
 *    ONE cooperative launch.  Every rank writes each 16-byte group of its
 *    input as LL lines [4 B value | 4 B flag] into its owner's receive area;
 *    the owner polls until every line's flag is current, reduces in rank
 *    order, rounds once and writes the result as LL lines into every rank's
 *    receive area; every rank polls those and stores its output.  Workspace:
 *    coll_all_reduce_workspace_size() bytes (256 + 4 N^2 seg size-of-dtype),
 *    256-byte aligned, zero-filled once before its first use, one call at a
 *    time; header as RING_LL (call counter, status pair at byte offset 16,
 *    COLL_DEV_TIMEOUT if a bounded poll ran out).  The counter occupies the
 *    flag's upper 30 bits: one fill serves COLL_TWOSHOT_LL_CALLS_PER_FILL
 *    calls, and a later call only raises COLL_DEV_EPOCH_WRAP, as in RING_LL.
 *    Buffers that are not
 *    16-byte aligned take the TWOSHOT kernel.  Needs N x (CTAs per SM) to
 *    fit on the GPU at once (COLL_ERR_UNSUPPORTED otherwise).
 *  TWOSHOT_LL128 ([RLL] "Traditional LL Protocols": the [120 B data | 8 B
 *    flag] line): TWOSHOT_LL with LL128 lines, 1.07 bytes per payload byte
 *    instead of 2.  A warp moves 4 lines at a time; the 8 stores of a line
 *    are not assumed to land together: its writer stores the data, fences
 *    (gpu scope) and then the flag, and its reader polls the flag, fences,
 *    and only then reads the data.  Bit-identical to TWOSHOT.  Workspace:
 *    coll_all_reduce_workspace_size() bytes, 256-byte aligned, zero-filled
 *    once, one call at a time, the same header (call counter, status pair,
 *    COLL_TWOSHOT_LL_CALLS_PER_FILL calls per fill).  Unaligned buffers take
 *    the TWOSHOT kernel.
 *  AUTO picks the form measured fastest on B200 for N and the bytes per rank
 *    (1 KiB .. 256 MiB per rank at 2, 3, 4 and 8 ranks, every one-launch
 *    form): ONESHOT for N == 3 up to 256 KiB and for N == 4 up to 64 KiB
 *    per rank, TWOSHOT otherwise, and TWOSHOT for any in-place call (ONESHOT
 *    cannot run in place).  Both give the rank-order result, so AUTO's bits
 *    do not depend on the choice.  ONESHOT and TWOSHOT ignore `workspace`.
 * In place (recv[r] == send[r]) is allowed for every algorithm but ONESHOT. */
COLL_API int coll_all_reduce(const void* const* send, void* const* recv, int nranks, size_t count,
                    coll_dtype_t dtype, coll_op_t op, coll_algo_t algo, void* workspace,
                    size_t workspace_bytes, coll_stream_t stream);
COLL_API size_t coll_all_reduce_workspace_size(int nranks, size_t count, coll_dtype_t dtype,
                                      coll_algo_t algo);
/* The form coll_all_reduce() runs for these arguments when nranks >= 2 and
 * count >= 1: ONESHOT, TWOSHOT, TWOSHOT_LL, TWOSHOT_LL128, RING_LL,
 * RING_CLUSTER, RING_CTA, RING_LANE, RING_WIRE or RING_STEPS (AUTO and RING
 * resolved, AUTO for a call that is not in place; `aligned` != 0 when every
 * buffer is 16-byte aligned).  RING_STEPS launches 2(N-1) kernels, the
 * others one.  Returns a negative COLL_ERR_* for an invalid rank count,
 * dtype or algo, and COLL_ERR_UNSUPPORTED for a RING_WIRE call that cannot
 * run.  Library introspection; the sources have no counterpart. */
COLL_API int coll_all_reduce_form(int nranks, size_t count, coll_dtype_t dtype, coll_algo_t algo,
                                  int aligned);

/* AllGather ([TUT] 7.1, 7.3): every recv[q] (N * send_count elements) gets
 * recv[q][r * send_count + i] = send[r][i]: the slices are concatenated, not
 * added.  In place: send[r] may be block r of recv[r]. */
COLL_API int coll_all_gather(const void* const* send, void* const* recv, int nranks, size_t send_count,
                    coll_dtype_t dtype, coll_stream_t stream);

/* All-to-All with equal blocks ([TUT] 8.1; [A2A] all_to_all_single): send[s]
 * is laid out [to 0, to 1, ..., to N-1], each block `count` elements;
 * afterwards recv[d] = [from 0, from 1, ..., from N-1].  N == 1 is a copy.
 * No overlap allowed. */
COLL_API int coll_all_to_all(const void* const* send, void* const* recv, int nranks, size_t count,
                    coll_dtype_t dtype, coll_stream_t stream);

/* All-to-All-v ([TUT] 8.2): per-pair lengths differ.  Rows are `row_elems`
 * elements.  Host arrays, N*N int64 each:
 *   send_counts[s*N + d]  rows rank s sends to rank d,
 *   send_displs[s*N + d]  first such row in send[s],
 *   recv_displs[d*N + s]  first row where they land in recv[d].
 * recv_capacity (host, N entries, rows) and send_capacity (host, N entries)
 * bound every block; either may be NULL to skip that check.  Rows of recv
 * not covered by any block are left untouched.  No overlap allowed. */
COLL_API int coll_all_to_all_v(const void* const* send, void* const* recv, int nranks,
                      const int64_t* send_counts, const int64_t* send_displs,
                      const int64_t* recv_displs, const int64_t* send_capacity,
                      const int64_t* recv_capacity, size_t row_elems, coll_dtype_t dtype,
                      coll_stream_t stream);

/* ------------------------------------------------------------------------
 * LL / LL128 packets ([RLL] "Traditional LL Protocols"; the receive side of
 * "Pro5000 ?").
 *   LL line    = 8 bytes:   u32 data word (message bytes 4L..4L+3, the last
 *                           word zero-padded) then u32 flag = (u32)step.
 *   LL128 line = 128 bytes: message bytes 120L..120L+119 (zero-padded at the
 *                           end) then u64 flag = step at bytes 120..127.
 * Little endian.  step >= 1 (and (u32)step != 0 for LL), so that zeroed
 * memory never validates.  coll_packed_bytes() gives the packed size:
 * 8*ceil(bytes/4), 128*ceil(bytes/120), or `bytes` for SIMPLE.
 * ------------------------------------------------------------------------ */
COLL_API size_t coll_packed_bytes(size_t bytes, coll_proto_t proto);

/* Encode `bytes` bytes of `src` into coll_packed_bytes(bytes, proto) bytes
 * at `packed`.  No overlap allowed.  Long 16-byte aligned LL messages go
 * through shared memory with bulk copies, whose waits are bounded (~2 s); a
 * wait that ran out (never seen) would leave the packet incomplete, and the
 * unpack of it reports the lines whose flags are wrong. */
COLL_API int coll_ll_pack(const void* src, void* packed, size_t bytes, coll_proto_t proto,
                 uint64_t step, coll_stream_t stream);

/* Decode into exactly `bytes` bytes at `dst`.  Every line whose flag is not
 * `step` adds 1 to d_status[1] (code COLL_DEV_FLAG_MISMATCH); its data is
 * still written.  d_status may be NULL. */
COLL_API int coll_ll_unpack(const void* packed, void* dst, size_t bytes, coll_proto_t proto,
                   uint64_t step, int* d_status, coll_stream_t stream);

/* The same two codecs for the equally long messages of all N virtual ranks
 * in one launch ([RLL] "Pro5000 ?": every rank encodes its own message
 * before the exchange and decodes the result after it): rank r's `bytes`
 * bytes at src[r] into packed[r], or packed[r] into dst[r].  Each result is
 * bit-identical to the one-rank call on that rank's buffers.  No message may
 * overlap any packet buffer, and the buffers written (packed[] for pack,
 * dst[] for unpack) must be disjoint; every packed[r] 16-byte aligned.
 * Unpack counts flag mismatches over all ranks into d_status[1]. */
COLL_API int coll_ll_pack_ranks(const void* const* src, void* const* packed, int nranks, size_t bytes,
                                coll_proto_t proto, uint64_t step, coll_stream_t stream);
COLL_API int coll_ll_unpack_ranks(const void* const* packed, void* const* dst, int nranks, size_t bytes,
                                  coll_proto_t proto, uint64_t step, int* d_status, coll_stream_t stream);

/* Packetised AllReduce: packed_in[r] are rank r's packets (proto, `count`
 * elements of payload, flag = step).  The kernel checks every input line's
 * flag (mismatches counted as above, over all ranks), reduces the payload in
 * rank order, and writes the result as packets with flag = step to every
 * packed_out[q].  Padding in the last line is written as zero.  In place
 * (packed_out[r] == packed_in[r]) is allowed.  proto SIMPLE is
 * coll_all_reduce(..., TWOSHOT). */
COLL_API int coll_all_reduce_packed(const void* const* packed_in, void* const* packed_out, int nranks,
                           size_t count, coll_dtype_t dtype, coll_op_t op, coll_proto_t proto,
                           uint64_t step, int* d_status, coll_stream_t stream);

/* ------------------------------------------------------------------------
 * MoE expert-parallel dispatch / combine ([TUT] 8.4, 8.5.1).  Experts are
 * spread evenly: expert e lives on rank e / (n_experts / N).  Every source
 * rank s has `tokens` tokens and, per token, `topk` distinct expert ids
 * (int32 [tokens, topk], row-major).  One row is sent per (token, expert).
 * Send order on a source: destination rank, then expert id, then token
 * index; receive order on a destination: source rank, then the sender's
 * order ([TUT] 8.1).  n_experts <= COLL_MAX_EXPERTS and divisible by N;
 * N * tokens * topk < 2^31.
 * ------------------------------------------------------------------------ */

/* Route: counts, prefix scans and the receive row of every pair.
 * Outputs (device): d_send_counts[s*N+d], d_send_displs[s*N+d],
 * d_recv_displs[d*N+s] (int64, rows) and, per source s, d_pos[s][t*topk+k]
 * (int32), the row of recv[expert / (n_experts/N)] that pair (t, k) is
 * written to.  A bad expert id raises COLL_DEV_BAD_ROUTE (positions are then
 * unspecified).  Deterministic: no result depends on atomics' order.
 * workspace: coll_moe_route_workspace_size() bytes, 256-byte aligned. */
COLL_API int coll_moe_route(const int32_t* const* topk_ids, int nranks, int tokens, int topk,
                   int n_experts, int64_t* d_send_counts, int64_t* d_send_displs,
                   int64_t* d_recv_displs, int32_t* const* d_pos, int* d_status,
                   void* workspace, size_t workspace_bytes, coll_stream_t stream);
COLL_API size_t coll_moe_route_workspace_size(int nranks, int tokens, int topk, int n_experts);

/* Route deduplicated per (token, destination rank) ([TUT] 8.5.1 names
 * dispatch designs that send a token once per rank it must reach; the
 * tutorial gives no layout, so this one is the plainest): one row per
 * (token, destination rank), so d_send_counts[s*N+d] is the number of tokens
 * of source s with at least one chosen expert on rank d.  Send order on a
 * source: destination rank, then token index; receive order as above.
 * d_pos[s][t*topk+k] is the row of (t, rank of expert k): the same row for
 * every k whose experts share a rank.  Dispatch and combine take these
 * positions unchanged; dispatch writes a row reached by several choices
 * once.  A repeated or out-of-range expert id raises COLL_DEV_BAD_ROUTE.
 * Same arguments and workspace (coll_moe_route_workspace_size()) as
 * coll_moe_route. */
COLL_API int coll_moe_route_dedup(const int32_t* const* topk_ids, int nranks, int tokens, int topk,
                         int n_experts, int64_t* d_send_counts, int64_t* d_send_displs,
                         int64_t* d_recv_displs, int32_t* const* d_pos, int* d_status,
                         void* workspace, size_t workspace_bytes, coll_stream_t stream);

/* Dispatch (the permute and the all-to-all-v in one pass): for every source
 * s, token t and choice k, recv[d][d_pos[s][t*topk+k]] = x[s][t], a row of
 * `hidden` elements, d = topk_ids[s][t][k] / (n_experts/N).  Each token row
 * is read once, and written once per distinct receive row (choices of a
 * token that share a row, as a deduplicated route gives them, share the
 * write).  Rows at or beyond recv_capacity_rows are not written and raise
 * COLL_DEV_SPLIT_OVERFLOW.  Bit copy. */
COLL_API int coll_moe_dispatch(const void* const* x, const int32_t* const* topk_ids,
                      const int32_t* const* d_pos, void* const* recv, int nranks, int tokens,
                      int topk, int n_experts, size_t hidden, coll_dtype_t dtype,
                      int64_t recv_capacity_rows, int* d_status, coll_stream_t stream);

/* Combine (the return all-to-all-v and the weighted sum in one pass):
 * out[s][t] = round( sum over k ascending of w[s][t][k] * y[d][d_pos] ) with
 * acc = fl32(w_0 * y_0), acc = fl32(acc + fl32(w_k * y_k)), one rounding to
 * dtype.  y[d] are the expert outputs in the receive layout of dispatch;
 * topk_w[s] is fp32 [tokens, topk].  Out-of-range rows raise
 * COLL_DEV_SPLIT_OVERFLOW and count as zero.  dtype BF16, FP16 or FP32. */
COLL_API int coll_moe_combine(const void* const* y, const int32_t* const* topk_ids,
                     const int32_t* const* d_pos, const float* const* topk_w, void* const* out,
                     int nranks, int tokens, int topk, int n_experts, size_t hidden,
                     coll_dtype_t dtype, int64_t recv_capacity_rows, int* d_status,
                     coll_stream_t stream);

/* ------------------------------------------------------------------------
 * All-reduce for callers that cannot allocate device memory.  The pages have
 * no counterpart of this entry point: it exists for code that is handed only
 * the ranks' buffers and may not call cudaMalloc -- a plug-in inside a host
 * framework that owns every byte of device memory through its own pool, or a
 * process whose memory was fully reserved (for example by a KV-cache pool) at
 * start-up, so that any further allocation fails.
 *
 * It is the RING algorithm of coll_all_reduce, with the same result bit for
 * bit, but its scratch (the fp32 / int32 partial sums that travel round the
 * ring) lives in a fixed array of COLL_RING_NOALLOC_SCRATCH_BYTES compiled
 * into this library: every GPU that loads the library holds that array until
 * the process exits.  No cudaMalloc, cudaFree or other allocating routine is
 * called.
 *  - count may be at most COLL_RING_NOALLOC_MAX_COUNT elements; larger
 *    calls return COLL_ERR_WORKSPACE and enqueue nothing.
 *  - The first call on a device (with that device current) looks up the
 *    array's device address; make that first call before any stream capture.
 *    Under lazy module loading (CUDA_MODULE_LOADING=LAZY, the default since
 *    CUDA 12.2) that lookup is also when the driver places the array on the
 *    device, so a process that reserves all of its device memory up front
 *    should make one call first -- a call with count == 0 is enough, since
 *    the lookup comes before every shortcut -- or run with
 *    CUDA_MODULE_LOADING=EAGER, which places the array when the library's
 *    kernels are loaded.
 *  - All calls share the one array, so calls whose work overlaps on the GPU
 *    (other streams, other threads) race: serialise them.  The array keeps
 *    the last call's partials; nothing in it needs to start at zero, because
 *    every partial is written before it is read.
 * In place (recv[r] == send[r]) is allowed. */
#define COLL_RING_NOALLOC_SCRATCH_BYTES (8u << 20)
#define COLL_RING_NOALLOC_MAX_COUNT (COLL_RING_NOALLOC_SCRATCH_BYTES / 4u)
COLL_API int coll_all_reduce_ring_noalloc(const void* const* send, void* const* recv, int nranks, size_t count,
                                          coll_dtype_t dtype, coll_op_t op, coll_stream_t stream);

/* ------------------------------------------------------------------------
 * Bounded wait on a device word (diagnostic).  Enqueues a one-thread kernel
 * that re-reads *flag until it equals `expect`, for at most `budget_us`
 * microseconds of GPU time; if the budget runs out it raises
 * COLL_DEV_TIMEOUT in d_status (required) and returns normally.  It is the
 * same bounded poll every waiting kernel of this library uses, exposed so that
 * the time-out path can be exercised on purpose with a flag that nothing
 * sets.  budget_us must be in [1, 10,000,000]. */
COLL_API int coll_wait_flag(const uint32_t* flag, uint32_t expect, uint32_t budget_us, int* d_status,
                            coll_stream_t stream);

/* ------------------------------------------------------------------------ */
COLL_API const char* coll_strerror(int status);
COLL_API int coll_version(void); /* major*10000 + minor*100 + patch */

#ifdef __cplusplus
} /* extern "C" */
#endif
#endif /* MVR_COLL_H */
