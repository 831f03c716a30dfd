/*
 * moe.h -- C ABI of one DwarfStar-quantised DeepSeek-V4-Flash MoE FFN layer
 * on an NVIDIA B200 (sm_100a).
 *
 * The layer (source: "DeepSeek-V4-Flash one-token computation flow, Dwarf
 * Star q2", qiita.com/sukimaengineer/items/cd76fec76d49a098abed, section
 * "MoE FFN 部の中身: router → top-6 → expert → 加重和"):
 *
 *   z = W_r x                      (F16 router, 4096 -> 256)
 *   s = sqrt(softplus(z))          (sqrtsoftplus scoring)
 *   top-k experts by s + bias      (bias for selection only; ties -> lower id)
 *   g_i = s_i / sum_sel s          (norm_topk_prob), w_i = routed_scaling * g_i
 *   y = shared(x) + sum_i w_i E_i(x),  E(x) = W_down (SiLU(W_gate x) * (W_up x))
 *
 * Hash-routed layers (the first three) skip the router: the expert ids come
 * from a token-id table and every selected expert gets routed_scaling / k.
 *
 * Weight formats ("2bit 量子化はなぜ「冗談ではない」のか", ds4.c を読み解く #2,
 * qiita.com/yoshiyakato/items/4678be0e7860ddb444ec, sections 3 and 4; and the
 * bit-allocation table of the first page):
 *   routed gate/up  IQ2_XXS  256 elements in 66 bytes
 *   routed down     Q2_K     256 elements in 84 bytes
 *   shared expert   Q8_0     32 elements in 34 bytes
 *   router          F16      [n_experts][hidden]
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library allocates no device memory: persistent state lives in the
 *     caller's `persist` buffer, per-call temporaries in `scratch`.
 *   - Every call is asynchronous on the given stream and never synchronises
 *     the host, except moe_poll_device_error.
 *   - A handle belongs to the device that is current at moe_init; moe_route
 *     and the forward calls return MOE_ERR_INVALID_ARG when another device
 *     is current.
 *   - Argument and shape errors are returned synchronously as a negative
 *     moe_status and described by moe_last_error() (thread-local).  No C++
 *     exception crosses this boundary.  Device-side problems (a bounded wait
 *     that ran out) are recorded in a device error word read back by
 *     moe_poll_device_error.
 *   - Layouts are row-major; packed weight matrices are [out_row][in_block],
 *     routed ones stacked as [expert][out_row][in_block].
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,       /* null pointer, negative count, bad enum */
  MOE_ERR_UNSUPPORTED_SHAPE = -2, /* dimensions this build does not handle */
  MOE_ERR_MISALIGNED = -3,        /* a pointer is not 16-byte aligned */
  MOE_ERR_WORKSPACE_TOO_SMALL = -4,
  MOE_ERR_CUDA = -5,              /* a CUDA runtime call failed */
  MOE_ERR_TIMEOUT = -6,           /* a bounded device wait ran out */
  MOE_ERR_DEVICE_FAULT = -7       /* the device reported another error */
} moe_status;

typedef enum { MOE_ROUTE_ROUTER = 0, MOE_ROUTE_HASH = 1 } moe_route_mode;

/* flags */
#define MOE_FLAG_PRENORM_RESIDUAL 1 /* forward computes x + MoE(RMSNorm(x)) */
/* calls above MOE_SMALL_T_MAX tokens add the routed experts' outputs in a fixed
 * order (each pair's weighted output in its own row of scratch, then every
 * token's rows summed in ascending expert id), so repeated calls give the same
 * bits; without it they are added with atomics in arrival order.  Costs
 * T*k*H*4 bytes of scratch (403 MB at T = 4096) and their write and read.
 * The small-token path is deterministic either way. */
#define MOE_FLAG_DETERMINISTIC 8
/* handles for expert parallelism (the moe_ep_* calls below); neither serves
 * moe_ffn_forward */
#define MOE_FLAG_EXPERTS_ONLY 2 /* a shard of routed experts: only the routed expert weights are read */
#define MOE_FLAG_NO_ROUTED 4    /* router (or table) and shared expert only: routed expert pointers may be NULL */

#define MOE_SMALL_T_MAX 32 /* largest T served by the small-token kernels */
#define MOE_CHUNKED_T_MAX 64 /* q2 layers: up to this T, the small-token kernels run on 32 tokens, then the rest */

/* formats of the routed experts (moe_config.routed_format) */
#define MOE_ROUTED_Q2 0  /* the q2 build: gate/up IQ2_XXS, down Q2_K */
#define MOE_ROUTED_Q4K 1 /* the q2-q4 build's upgraded layers: gate, up and down Q4_K (144 bytes per 256) */

/* block formats of moe_quantize */
#define MOE_QUANT_Q8_0 0 /* 32 values in 34 bytes */
#define MOE_QUANT_Q2_K 1 /* 256 values in 84 bytes */
#define MOE_QUANT_Q4_K 2 /* 256 values in 144 bytes (the Q4_K layout of MOE_ROUTED_Q4K) */

typedef struct {
  int hidden;           /* H: multiple of 256 (4096 for V4-Flash) */
  int inter;            /* I: routed expert intermediate, multiple of 256 (2048) */
  int n_experts;        /* E: routed experts, k <= E <= 256 */
  int top_k;            /* k: 1..8 (6) */
  int shared_inter;     /* Is: shared expert intermediate, multiple of 256 (2048) */
  int vocab;            /* rows of tid2eid (hash mode; 129280 for V4-Flash) */
  float routed_scaling; /* 1.5 */
  float rms_eps;        /* RMSNorm epsilon when MOE_FLAG_PRENORM_RESIDUAL is set (1e-6) */
  int mode;             /* moe_route_mode */
  int flags;            /* MOE_FLAG_* */
  int routed_format;    /* MOE_ROUTED_*; MOE_ROUTED_Q4K layers do not run moe_ffn_forward_noalloc */
} moe_config;

typedef struct {
  const void *router_w_f16;   /* [E][H] IEEE f16; NULL in hash mode */
  const float *router_bias;   /* [E] fp32 selection bias; NULL in hash mode */
  const int32_t *tid2eid;     /* [vocab][k] expert ids; NULL in router mode */
  const void *gate_iq2xxs;    /* [E][I][H/256] 66-byte blocks (144-byte Q4_K blocks with MOE_ROUTED_Q4K) */
  const void *up_iq2xxs;      /* [E][I][H/256] 66-byte blocks (Q4_K likewise) */
  const void *down_q2k;       /* [E][H][I/256] 84-byte blocks (Q4_K likewise) */
  const void *sh_gate_q80;    /* [Is][H/32] 34-byte blocks */
  const void *sh_up_q80;      /* [Is][H/32] 34-byte blocks */
  const void *sh_down_q80;    /* [H][Is/32] 34-byte blocks */
  const uint8_t *iq2_grid;    /* [256][8] codebook; every entry must be <= 127 (may be NULL with MOE_ROUTED_Q4K) */
} moe_weights;

typedef struct moe_handle moe_handle;

/*
 * Sizes of the two caller-owned buffers for calls with up to `max_tokens`
 * tokens.  `persist` must outlive the handle; `scratch` is needed only for
 * the duration of each call (stream order).  Either output may be NULL.
 */
moe_status moe_workspace_size(const moe_config *cfg, int max_tokens, size_t *persist_bytes,
                              size_t *scratch_bytes);

/*
 * Validates the configuration and the weight pointers (non-null as the mode
 * requires, 16-byte aligned), records them in a host-side handle and
 * enqueues the initialisation of `persist` on `stream` (it checks the
 * codebook range into the device error word, computes the router rows'
 * norms, and copies the tensor maps through which the batched path's
 * tensor-memory-access unit reads the routed weight tiles).  The weight
 * buffers are read, never written, and must stay valid and unchanged while
 * the handle is used.
 *
 * Two environment variables, read here, select equivalent forms of the
 * batched path (same results, for comparison and testing): MOE_GEMM_TMA set
 * to "0" has its producer warps load the packed weight tiles themselves
 * instead of through tensor copies; MOE_SHARED_DENSE set to "0" keeps the
 * shared expert on per-tile Q8_0 decoding at every token count.
 *
 * Hash mode: every row of tid2eid must hold top_k distinct expert ids in
 * [0, n_experts) (the kernels index the expert weights with them and count
 * each selected expert once per token).  moe_init checks the whole table on
 * `stream` and waits for that check (the one synchronisation of this call);
 * a row that breaks the rule returns MOE_ERR_INVALID_ARG naming the row, and
 * no handle is created.
 */
moe_status moe_init(const moe_config *cfg, const moe_weights *w, void *persist, size_t persist_bytes,
                    moe_stream_t stream, moe_handle **out);

/*
 * Routing only.  x: [T][H] fp32 (device).  token_ids: [T] int32 (hash mode;
 * ignored in router mode, may be NULL there).  Writes idx [T][k] int32 with
 * each row's expert ids in ascending order and w [T][k] fp32 routing weights
 * in the same order (each row sums to routed_scaling).  When both
 * expert_offsets ([E+1]) and perm ([T*k]) are non-NULL it also writes the
 * grouping of the T*k (token, slot) pairs by expert: offsets[e] is the
 * number of pairs on experts below e, and perm lists t*k + slot for each
 * expert in ascending token order.  With MOE_FLAG_PRENORM_RESIDUAL the
 * router sees RMSNorm(x).
 */
moe_status moe_route(moe_handle *h, const float *x, const int32_t *token_ids, int T, int32_t *idx, float *w,
                     int32_t *expert_offsets, int32_t *perm, void *scratch, size_t scratch_bytes,
                     moe_stream_t stream);

/*
 * The whole layer.  x: [T][H] fp32 input; y: [T][H] fp32 output
 * (overwritten; may alias x only with MOE_FLAG_PRENORM_RESIDUAL, where
 * y = x + MoE(RMSNorm(x))).  T = 0 is a no-op.  Calls with
 * T <= MOE_SMALL_T_MAX run the small-token path (two kernel launches: input
 * preparation and router, then routing and every expert unit); q2 layers with
 * T <= MOE_CHUNKED_T_MAX run it twice, on the first MOE_SMALL_T_MAX tokens and
 * then on the rest (the same results per token); larger T the batched
 * tensor-core path (router, certificate, fix-up, permutation, the grouped
 * GEMMs, and from 257 tokens the shared expert's expansion and dense GEMMs).
 */
moe_status moe_ffn_forward(moe_handle *h, const float *x, const int32_t *token_ids, int T, float *y,
                           void *scratch, size_t scratch_bytes, moe_stream_t stream);

/*
 * moe_ffn_forward for callers that cannot allocate device memory.  (This
 * entry point has no counterpart in the source pages; it only changes where
 * the per-call temporaries live.)
 *
 * Some callers of this layer are not allowed to call cudaMalloc or any other
 * allocator: for example a plugin inside a serving engine or framework that
 * owns every device allocation through its own memory pool, or a program that
 * must keep a fixed device-memory plan once it has started.  Such a caller
 * can still hand over its inputs and outputs, but has no scratch buffer to
 * give.  This variant runs the same small-T kernels as moe_ffn_forward with
 * their scratch in a buffer built into the library: a 16 MiB array in device
 * global memory that every GPU loading the library holds until the process
 * exits.  Nothing is allocated by the call (no cudaMalloc, cudaFree or
 * allocating library routine).
 *
 * Limits: 1 <= T <= 8 tokens, and the layer's small-T scratch for T must fit
 * in 16 MiB (the V4-Flash shapes need about 6.2 MiB at T = 8); larger requests
 * return MOE_ERR_UNSUPPORTED_SHAPE or MOE_ERR_WORKSPACE_TOO_SMALL with a
 * message.  T = 0 is a no-op.  The current device must be the handle's
 * device.  Each call made outside stream capture looks up the buffer's device
 * address (cudaGetSymbolAddress, with that device current; the lookup also
 * follows the buffer after a cudaDeviceReset) and keeps it for calls made
 * while `stream` is being captured; make the first call on a device before
 * any stream capture.  Every call on a device shares the one
 * buffer and leaves its contents behind; the kernels clear the counters they
 * need at the start of each call.  Calls whose executions overlap on the GPU
 * (different streams, or different handles on the same device) race on the
 * buffer: order them on one stream or synchronise between them.
 * Arguments and errors are as for moe_ffn_forward.
 */
moe_status moe_ffn_forward_noalloc(moe_handle *h, const float *x, const int32_t *token_ids, int T, float *y,
                                   moe_stream_t stream);

/* Synchronises `stream`, then returns and clears the device error word:
 * MOE_OK, MOE_ERR_TIMEOUT, MOE_ERR_UNSUPPORTED_SHAPE (codebook entry > 127)
 * or MOE_ERR_DEVICE_FAULT. */
moe_status moe_poll_device_error(moe_handle *h, moe_stream_t stream);

/* Human-readable description of the last error on this thread ("" if none). */
const char *moe_last_error(void);

/*
 * Optional instrumentation.  While set, every moe_ffn_forward on this handle
 * records `ev_begin` on its stream right before the layer's dominant kernel
 * (the routed gate/up kernel) and `ev_end` right after it.  Both are
 * cudaEvent_t handles created and owned by the caller; pass NULL for both to
 * stop recording.  Recording changes no work the layer does.
 */
moe_status moe_set_timing_events(moe_handle *h, void *ev_begin, void *ev_end);

/*
 * Stacked layers (x <- x + MoE_l(RMSNorm(x)) for l = 0, 1, ...; "DeepSeek-
 * V4-Flash one-token computation flow", block structure): after
 * moe_set_next_layer(h, next), every small-token forward on h brings the
 * weights that `next` reads first -- its router rows and its shared
 * expert's gate and up rows -- into the L2 cache near the end of h's expert
 * kernel, so that the next layer's router and shared-expert work start from
 * L2 rather than HBM.  A prefetch changes no result.  `next` must stay
 * valid while h is used (NULL clears it).  Records pointers only.
 */
moe_status moe_set_next_layer(moe_handle *h, const moe_handle *next);

/*
 * Test hook for the device-side error path.  The kernels bound every wait on
 * work of other warps or blocks (a down-projection unit waiting for the
 * SwiGLU slice it reads, a warp waiting for its block's routing table, the
 * hand-offs between the tensor-core kernel's producer, MMA and epilogue
 * roles) at about 2 s; this sets that bound to `cycles` SM clock cycles for
 * the later calls on this handle (0 restores the default).  A wait that runs
 * out records MOE_ERR_TIMEOUT in the device error word and the kernel goes
 * on or leaves without waiting further on others: it still waits for its
 * own in-flight copies and tensor-core work (with the default bound), frees
 * its tensor memory and returns, so the context stays usable.  That call's
 * output is undefined; the next call starts from clean counters.
 */
moe_status moe_set_wait_limit(moe_handle *h, long long cycles);

/*
 * Offline encoder: n fp32 values -> blocks of `format` (MOE_QUANT_Q8_0: n a
 * multiple of 32, n/32 blocks of 34 bytes; MOE_QUANT_Q2_K / MOE_QUANT_Q4_K: n
 * a multiple of 256, n/256 blocks of 84 / 144 bytes), the writer side of the
 * formats the layer
 * reads ("2bit 量子化はなぜ「冗談ではない」のか", section 3: per 16-element
 * sub-block a scale and a min, codes 0..3, the page's packing; "DeepSeek-V4-
 * Flash one-token computation flow", section "Dwarf Star の量子化の工夫": Q8_0
 * has one symmetric scale per 32 values).  The estimator is plain min/max with
 * every decision in IEEE binary32, round to nearest even; the steps are listed
 * in csrc/quant.cu.  x and out are device pointers, 16-byte aligned; a matrix
 * of rows whose length is a multiple of the block size is encoded row after
 * row by passing it whole.  nonfinite_blocks (device int32, may be NULL) is
 * incremented once per block that holds a NaN or an infinity; such blocks are
 * written as zeros.  Asynchronous on `stream`; n = 0 is a no-op.
 */
moe_status moe_quantize(int format, const float *x, int64_t n, void *out, int32_t *nonfinite_blocks,
                        moe_stream_t stream);

/*
 * Expert parallelism: the routed experts of a layer split over G ranks (one
 * GPU each) in contiguous blocks of E/G experts; rank r owns global ids
 * [r*E/G, (r+1)*E/G).  The exchange itself (two all-to-alls of rows between
 * ranks) is the caller's, e.g. NCCL through torch.distributed; these calls do
 * the work on each side of it.  The pages' counterpart is ds4's mode that
 * splits one model over two machines ("DeepSeek-V4-Flash one-token
 * computation flow", section "128GB にどう収めるか"); the split by experts is
 * this library's choice.  The calls run the batched (tensor-core) kernels
 * for any T.
 *
 *   1. moe_ep_dispatch (every rank, on its own T tokens, with a handle that
 *      has the router or table and the shared expert; MOE_FLAG_NO_ROUTED lets
 *      it hold no routed weights): routing, then the T*k (token, slot) pairs
 *      grouped by expert as moe_route gives them (expert_offsets [E+1], perm
 *      [T*k]), and for pair perm[i], in row i: x_send [T*k][H] the expert
 *      input as IEEE f16 (RMSNorm(x) with MOE_FLAG_PRENORM_RESIDUAL, else x),
 *      e_send [T*k] the global expert id, w_send [T*k] the routing weight.
 *      The rows for rank r are expert_offsets[r*E/G] .. expert_offsets[(r+1)*E/G].
 *   2. (exchange: each rank receives the rows for its experts from all ranks)
 *   3. moe_ep_experts (on the shard handle: MOE_FLAG_EXPERTS_ONLY, n_experts
 *      = the shard's E/G, routed weight arrays holding only the shard's
 *      experts, first_expert = the shard's first global id): for the N
 *      received rows, out[i] = w_recv[i] * E_{e_recv[i]}(x_recv[i]) (fp32
 *      [N][H]).  A row whose id is outside the shard gets zeros and records
 *      MOE_ERR_INVALID_ARG in the device error word.
 *   4. (exchange back: the out rows return to the rank and row they came from)
 *   5. moe_ep_combine (the dispatching rank): y [T][H] = shared expert (plus x
 *      with MOE_FLAG_PRENORM_RESIDUAL) + for each token the sum over its k
 *      pairs, in ascending expert id, of out_back rows (row i for pair
 *      perm[i]).  y may alias x only with MOE_FLAG_PRENORM_RESIDUAL.
 *
 * moe_ep_workspace_size gives each call's scratch for up to max_tokens tokens
 * and max_recv_rows received rows.  All pointers are device pointers, 16-byte
 * aligned where they hold rows; every call is asynchronous on `stream`.
 */
moe_status moe_ep_workspace_size(const moe_config *cfg, int max_tokens, int max_recv_rows, size_t *dispatch_bytes,
                                 size_t *experts_bytes, size_t *combine_bytes);
moe_status moe_ep_dispatch(moe_handle *h, const float *x, const int32_t *token_ids, int T, int32_t *expert_offsets,
                           int32_t *perm, void *x_send, int32_t *e_send, float *w_send, void *scratch,
                           size_t scratch_bytes, moe_stream_t stream);
moe_status moe_ep_experts(moe_handle *shard, const void *x_recv, const int32_t *e_recv, const float *w_recv, int N,
                          int first_expert, float *out, void *scratch, size_t scratch_bytes, moe_stream_t stream);
moe_status moe_ep_combine(moe_handle *h, const float *x, int T, const int32_t *perm, const float *out_back, float *y,
                          void *scratch, size_t scratch_bytes, moe_stream_t stream);

/* Frees the host-side handle (the caller frees `persist`). NULL is a no-op. */
void moe_destroy(moe_handle *h);

#ifdef __cplusplus
}
#endif
#endif
