/*
 * mtgr.h — C ABI of libmtgr.so: the forward pass of the MTGR HSTU block and
 * block stack over user-aggregated, jagged token sequences, for NVIDIA B200
 * (sm_100a).
 *
 * Method: "MTGR: Industrial-Scale Generative Recommendation Framework in
 * Meituan" (summary page, section "Method"; fun-rec "MTGR: Hybrid Paradigm
 * Modeling", 7.3.1 data organisation, 7.3.3 Group Layer Normalization,
 * 7.3.4 Dynamic Masking). Each user request is one sample
 * D = [U, S, R, [C,I]_1..K]; users are packed back to back; one HSTU block is
 *   X~ = GroupLN_1(X);  Q|K|V|U = X~ W_qkvu^T
 *   G  = (silu(Q K^T) (.) M / N) V (.) U          (per head, no 1/sqrt(dh))
 *   X  <- MLP(GroupLN_2(G)) + X,   MLP = Linear -> SiLU -> Linear
 * with the three-rule mask M and N the user's total token count.
 *
 * Around the stack:
 *  - the per-domain token MLPs that build X (mtgr_tokenize);
 *  - the CTR/CTCVR heads on the candidates' output rows
 *    (mtgr_candidate_heads);
 *  - serving with each layer's Q|K|V|U of the users' contexts cached, the
 *    candidates then scored against it (mtgr_stack_fwd_rows,
 *    mtgr_stack_fwd_candidates);
 *  - two block variants the pages leave open (mtgr_block_params.variant).
 *
 * Conventions shared by every entry point:
 *  - Pointers named d_* are DEVICE pointers (CUDA global memory) on the
 *    current device; the caller owns and frees all memory. The library never
 *    allocates or frees device memory and keeps no state between calls other
 *    than cached device attributes.
 *  - All work is enqueued asynchronously on the given stream (a cudaStream_t;
 *    NULL is the legacy default stream). Entry points do not synchronise.
 *  - Return value: MTGR_OK or an error code for errors the host can see
 *    (bad arguments, unsupported shapes, launch failures). Errors that depend
 *    on device data (inconsistent lengths, capacity overflow, an internal
 *    wait that timed out) are written to the caller's device status word
 *    (int32, 0 = ok; the first error wins) and must be read after the stream
 *    is synchronised. No entry point prints, traps or throws.
 *  - Token layout: user b occupies rows [user_off[b], user_off[b+1]) in the
 *    order U, S, R, C. Group ids: 0 = U, 1 = S, 2 = R, 3 = C.
 *  - Timestamps are int64, one per token; entries of U tokens are ignored.
 *  - Thread safety: calls on different streams may run concurrently; calls
 *    sharing a workspace must be ordered by the caller.
 */
#ifndef MTGR_H
#define MTGR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MTGR_API __attribute__((visibility("default")))

/* status codes */
#define MTGR_OK 0
#define MTGR_ERR_INVALID_ARG 1        /* null pointer, bad size or inconsistent argument */
#define MTGR_ERR_CUDA 2               /* a CUDA runtime call or kernel launch failed */
#define MTGR_ERR_UNSUPPORTED 3        /* dtype / head size / architecture not supported */
#define MTGR_ERR_CAPACITY 4           /* an output or workspace buffer is too small */
#define MTGR_ERR_TIMEOUT 5            /* device: an internal wait exceeded its limit */
#define MTGR_ERR_DEVICE_VALIDATION 6  /* device: lengths negative or not summing to T */
#define MTGR_ERR_RANGE 7              /* device: a value left the range of an f16 intermediate
                                         (the Q|K|V|U projection or the attention's silu
                                         weights P, both above 65504 in magnitude) */

/* element types */
#define MTGR_F32 0
#define MTGR_BF16 1
#define MTGR_F16 2

/* canonical mask-metadata tile (rows x columns of the user-relative grid) */
#define MTGR_TILE_M 128
#define MTGR_TILE_N 128

typedef void* mtgr_stream_t; /* a cudaStream_t */

/* Human-readable name of a status code. Never returns NULL. */
MTGR_API const char* mtgr_status_string(int status);

/* Library ABI version (major * 100 + minor). */
MTGR_API int mtgr_version(void);

/*
 * Jagged packing (summary page, Method: D = [U, S, R, [C,I]_1..K]; chenhuiyu
 * blog: sequence packing keeps users from attending to one another).
 *   d_lens     [B][4] int32: N_U, N_S, N_R, K of each user (read)
 *   T          total token count the caller expects (= sum of d_lens)
 *   d_seg_off  [4B+1] int32: row where U, S, R, C of each user start; last = T
 *   d_user_off [B+1] int32
 *   d_group_id [T] int8
 *   d_status   device int32 status word (MTGR_ERR_DEVICE_VALIDATION when a
 *              length is negative or the lengths do not sum to T)
 * B = 0 is valid (writes seg_off[0] = user_off[0] = 0).
 */
MTGR_API int mtgr_pack_offsets(int32_t B, const int32_t* d_lens, int32_t T, int32_t* d_seg_off,
                               int32_t* d_user_off, int8_t* d_group_id, int32_t* d_status,
                               mtgr_stream_t stream);

/* Bytes of device workspace mtgr_build_mask_meta needs. */
MTGR_API size_t mtgr_mask_meta_workspace_bytes(int32_t q_capacity, int32_t kt_capacity);

/* One item of the attention's work list (64 bytes): up to two consecutive
 * q-tiles (qt0, qt0 + 1) of one user, which share every key/value tile load. */
typedef struct mtgr_work_item {
  int32_t us;       /* first row of the user */
  int32_t n;        /* user length N_b */
  int32_t n_u;      /* N_U */
  int32_t n_us;     /* N_U + N_S */
  int32_t c_lo;     /* N_U + N_S + N_R */
  int32_t qt0;      /* first q-tile of the pair (within the user) */
  int32_t b;        /* user index */
  int32_t nq;       /* q-tiles in the item: 1 or 2 */
  int32_t e0a, e1a; /* entries of q-tile qt0: [e0a, e1a) of the CSR */
  int32_t e0b, e1b; /* entries of q-tile qt0 + 1 (empty range when nq == 1) */
  int32_t n_union;  /* k-tiles non-empty for at least one of the two q-tiles */
  int32_t reserved;
  int64_t rt_base;  /* the user's first rank-table entry */
} mtgr_work_item;

/*
 * Mask metadata: the canonical list of non-empty 128x128 tiles of every
 * user's mask M (fun-rec 7.3.4 Rules 1-3; summary page, Method, mask rules).
 *   Rule 1: keys in U and S are visible to every query of the user.
 *   Rule 2: a key j in R is visible to query i iff t_j < t_i or j == i
 *           (U queries carry no time and never see R keys).
 *   Rule 3: a candidate key is visible only to itself.
 * Tiles lie on the user-relative grid (q-tile qt covers user rows
 * [128 qt, 128 qt + 128)); only cells inside the user count. A tile is EMPTY
 * (omitted) if no cell is visible, FULL if every cell is, PARTIAL otherwise.
 *   d_seg_off    [4B+1] from mtgr_pack_offsets
 *   d_ts         [T] int64 timestamps
 *   q_capacity   rows available in d_qtile_desc/d_order (>= sum ceil(N_b/128))
 *   kt_capacity  >= max_b ceil(N_b/128)
 *   e_capacity   entries available in d_entries
 *   d_qtile_desc [q_capacity][2] int32: (user, qt), user-major, qt ascending
 *   d_row_ptr    [q_capacity+1] int32: CSR row pointers into d_entries
 *   d_entries    [e_capacity] int32: (kt << 1) | partial, kt ascending per row
 *   d_order      [q_capacity] int32: the attention's work order: q-tiles user
 *                by user, users by descending length (ties by ascending user
 *                index), each user's q-tiles by ascending qt
 *   d_counts     [4] int64: Q (q-tiles), E (entries), visible (query,key) pairs,
 *                P (work items: q-tile pairs)
 *   rt_capacity  entries available in d_rt_mask (>= sum over users of
 *                G_b (N_R,b + 1), G_b = number of 64-column groups of the
 *                user's key range [N_U+N_S, N_U+N_S+N_R) that hold R keys)
 *   d_rt_cnt     [T] int32: cnt_i = number of R keys of token i's user with a
 *                timestamp strictly below t_i (0 for U tokens)
 *   d_rt_off     [B+1] int64: start of each user's rank tables in d_rt_mask
 *   d_rt_mask    [rt_capacity] uint64: rule 2 as prefix tables. With the
 *                user's R keys ordered by (timestamp, index), entry
 *                rt_off[b] + g (N_R + 1) + r holds the bits (column mod 64
 *                within the user-relative 64-column group N_U+N_S rounded down
 *                to 64, plus g) of the R keys ranked below r. R key j != i is
 *                visible to query i iff its bit is set in the entry at r = cnt_i.
 *   d_work       [q_capacity] mtgr_work_item: the work list, in work order:
 *                each user's q-tiles in pairs (qt 0-1, 2-3, ...), with the
 *                user's offsets and both CSR ranges (one load per item)
 *   d_ws, ws_bytes  workspace of mtgr_mask_meta_workspace_bytes() bytes
 *   d_status     device status word (MTGR_ERR_CAPACITY if Q, E, the rank
 *                tables or a user's tile count exceed the capacities, or a
 *                user has more than 4096 R tokens; no q-tile is then published)
 */
MTGR_API int mtgr_build_mask_meta(int32_t B, const int32_t* d_seg_off, const int64_t* d_ts,
                                  int32_t q_capacity, int32_t kt_capacity, int32_t e_capacity,
                                  int64_t rt_capacity, int32_t* d_qtile_desc, int32_t* d_row_ptr,
                                  int32_t* d_entries, int32_t* d_order, int64_t* d_counts,
                                  int32_t* d_rt_cnt, int64_t* d_rt_off, uint64_t* d_rt_mask,
                                  mtgr_work_item* d_work, void* d_ws, size_t ws_bytes,
                                  int32_t* d_status, mtgr_stream_t stream);

/*
 * mtgr_build_mask_meta without a caller-provided workspace, for callers that
 * cannot allocate device memory when they build a batch: for example a serving
 * process that hands all of its device memory to its own pool at start-up and
 * forbids later allocations (cudaMalloc/cudaFree can synchronise the device and
 * take unpredictable time), or a plain C host program that wants a fixed device
 * footprint. The paper has no counterpart; this is a deployment convenience.
 *
 * Same arguments and results as mtgr_build_mask_meta minus d_ws / ws_bytes.
 * The scratch (one byte per q-tile and k-tile) lives in a fixed array of
 * MTGR_STATIC_META_SCRATCH_BYTES (4 MiB) inside the library's own device
 * memory, which every GPU that loads the library holds until the process
 * exits. Limits and behaviour:
 *  - q_capacity * kt_capacity must not exceed MTGR_STATIC_META_SCRATCH_BYTES;
 *    larger batches return MTGR_ERR_CAPACITY without touching the device (use
 *    mtgr_build_mask_meta with your own workspace for those).
 *  - The first call in a CUDA context looks up the array's device address
 *    (once per context, with that context current) and, under CUDA's lazy
 *    module loading, is also the point where the driver loads the library's
 *    module and commits the 4 MiB array on that device. Make that first call
 *    (B = 0 is enough) at start-up, before the caller's memory pool takes the
 *    device's free memory and before any stream capture. A device reset or a
 *    new context (e.g. one the caller creates with the driver API) gets its
 *    own lookup on its first call.
 *  - It never calls cudaMalloc, cudaFree or any allocating routine.
 *  - All calls share the one array per device and it keeps the last call's
 *    contents (every call overwrites what it reads, so nothing needs
 *    clearing). Calls whose work overlaps on the GPU — on different streams or
 *    from different host threads without ordering — race on it: order them.
 */
#define MTGR_STATIC_META_SCRATCH_BYTES (4u << 20)
MTGR_API int mtgr_build_mask_meta_static(int32_t B, const int32_t* d_seg_off, const int64_t* d_ts,
                                         int32_t q_capacity, int32_t kt_capacity,
                                         int32_t e_capacity, int64_t rt_capacity,
                                         int32_t* d_qtile_desc, int32_t* d_row_ptr,
                                         int32_t* d_entries, int32_t* d_order, int64_t* d_counts,
                                         int32_t* d_rt_cnt, int64_t* d_rt_off,
                                         uint64_t* d_rt_mask, mtgr_work_item* d_work,
                                         int32_t* d_status, mtgr_stream_t stream);

/*
 * Group-Layer Normalization (fun-rec 7.3.3, the GLN formula):
 *   y_i = (x_i - mean_i) / sqrt(var_i + eps) * gamma[g(i)] + beta[g(i)]
 * with mean and biased variance of token i over its d features and g(i) the
 * token's group id.
 *   x_dtype / y_dtype: (MTGR_F32, MTGR_F32), (MTGR_F32, MTGR_BF16) or
 *                      (MTGR_BF16, MTGR_BF16); x, y [T][d] row-major
 *   d_group_id [T] int8 in [0, G)
 *   d_gamma, d_beta [G][d] float32
 * d must be a multiple of 8 and at most 8192.
 */
MTGR_API int mtgr_group_layernorm(int32_t T, int32_t d, int32_t x_dtype, const void* d_x,
                                  const int8_t* d_group_id, int32_t G, const float* d_gamma,
                                  const float* d_beta, float eps, int32_t y_dtype, void* d_y,
                                  mtgr_stream_t stream);

/*
 * GroupLN with pooled statistics (MTGR_VARIANT_POOLED_GLN): for every user b
 * and group g, one mean and one biased variance over all N_{b,g} x d values of
 * rows [d_seg_off[4b+g], d_seg_off[4b+g+1]) (d_seg_off from
 * mtgr_pack_offsets, [4B+1], device); y = (x - mean) / sqrt(var + eps) *
 * gamma[g] + beta[g]. gamma, beta [4][d] float32; x, y [T][d] of x_dtype,
 * y_dtype (F32 -> F32, F32 -> BF16, BF16 -> BF16); d % 8 == 0.
 */
MTGR_API int mtgr_group_layernorm_pooled(int32_t B, const int32_t* d_seg_off, int32_t d,
                                         int32_t x_dtype, const void* d_x, const float* d_gamma,
                                         const float* d_beta, float eps, int32_t y_dtype, void* d_y,
                                         mtgr_stream_t stream);

/* A packed batch plus its mask metadata (all device pointers). */
typedef struct mtgr_batch {
  int32_t B;                  /* users */
  int32_t T;                  /* tokens */
  int32_t q_capacity;         /* rows of qtile_desc/order (launch bound, >= Q) */
  int32_t kt_capacity;        /* >= max_b ceil(N_b/128) */
  const int32_t* seg_off;     /* [4B+1] */
  const int32_t* user_off;    /* [B+1] */
  const int8_t* group_id;     /* [T] */
  const int64_t* ts;          /* [T] */
  const int32_t* qtile_desc;  /* [q_capacity][2] */
  const int32_t* row_ptr;     /* [q_capacity+1] */
  const int32_t* entries;     /* [E] */
  const int32_t* order;       /* [q_capacity] */
  const int64_t* counts;      /* [4] Q, E, visible pairs, P */
  const int32_t* rt_cnt;      /* [T] rank-table index of each token */
  const int64_t* rt_off;      /* [B+1] */
  const uint64_t* rt_mask;    /* rank tables of rule 2 */
  const mtgr_work_item* work; /* [q_capacity] work list */
  const float* norm;          /* optional [B] normaliser override; NULL = user length */
  int32_t* status;            /* device status word */
} mtgr_batch;

/*
 * Masked pointwise SiLU attention with the 1/N normaliser and the U gate
 * (summary page, Method: V~ = silu(K^T Q)/(N_U+N_S+N_R+N_I) M V; the gate
 * V~ (.) U of the block update):
 *   G[i, h] = (1/N_b) sum_j silu(q_i,h . k_j,h) M_ij v_j,h  (.)  u_i,h
 *   d_qkvu   [T][4d] row-major, column blocks Q | K | V | U, head h at
 *            columns [h dh, (h+1) dh) of each block; qkvu_dtype MTGR_BF16 or
 *            MTGR_F16 (tensor-core path, dh = 64) or MTGR_F32 (exact SIMT path,
 *            dh in {32, 64})
 *   d_g      [T][d] output, out_dtype MTGR_F32 or MTGR_BF16 (MTGR_F32 only for
 *            the f32 path)
 * The mask is evaluated tile by tile from the metadata and the timestamps and
 * is never stored. d = H * dh, d % 64 == 0 for the tensor-core path.
 */
MTGR_API int mtgr_hstu_attention_fwd(const mtgr_batch* batch, int32_t d, int32_t H,
                                     int32_t qkvu_dtype, const void* d_qkvu, int32_t out_dtype,
                                     void* d_g, mtgr_stream_t stream);

/*
 * Block variants, readings the pages leave open (flags of
 * mtgr_block_params.variant, bf16 blocks only; 0 is the block as the
 * summary page's Method writes it):
 *   MTGR_VARIANT_POOLED_GLN: both GroupLNs take one mean and one variance
 *     over all values of each (user, group) segment (the practice article's
 *     3.1 GLN pseudocode, group_mean = mean(group_hidden_states)). Not with
 *     mtgr_stack_fwd_rows on rows after 0 (MTGR_ERR_UNSUPPORTED).
 *   MTGR_VARIANT_SILU_QKVU: Q, K, V, U = silu(X~ W_qkvu^T + b), HSTU's
 *     pointwise SiLU on the projections (one reading of the blog posts'
 *     "HSTU-style SiLU attention and gating"; it also gates with silu(U)).
 *   MTGR_VARIANT_RAB: HSTU's relative attention bias, added to every score
 *     before the SiLU: silu(q_i . k_j + rab_h(i, j)) with
 *     rab_h(i, j) = rab_pos[h][clip(i - j, -MTGR_RAB_MAX_DIST,
 *     MTGR_RAB_MAX_DIST) + MTGR_RAB_MAX_DIST] + rab_time[h][b(|t_i - t_j|)],
 *     i, j the positions within the user, b(0) = 0 and b(dt) =
 *     min(floor(log2 dt) + 1, MTGR_RAB_TIME_BUCKETS - 1), and bucket 0 when
 *     either token is a U token (no time). The pages name this bias only
 *     through HSTU; this is the reading taken. Positions are those of the
 *     batch as given, so a candidate scored in a chunk of its own sees the
 *     position term of its place in that chunk.
 */
#define MTGR_VARIANT_POOLED_GLN 1
#define MTGR_VARIANT_SILU_QKVU 2
#define MTGR_VARIANT_RAB 4
#define MTGR_RAB_MAX_DIST 128
#define MTGR_RAB_TIME_BUCKETS 32

/* Parameters of one HSTU block (device pointers; PyTorch Linear [out][in] layout). */
typedef struct mtgr_block_params {
  int32_t d;                  /* d_model */
  int32_t H;                  /* heads, dh = d / H */
  int32_t d_ff;               /* MLP hidden width */
  int32_t dtype;              /* MTGR_BF16: bf16 weights, tensor cores; MTGR_F32: f32 SIMT */
  float eps;                  /* GroupLN epsilon */
  int32_t variant;            /* 0, or MTGR_VARIANT_* flags (bf16 only) */
  const float* gln1_gamma;    /* [4][d] */
  const float* gln1_beta;     /* [4][d] */
  const float* gln2_gamma;    /* [4][d] */
  const float* gln2_beta;     /* [4][d] */
  const void* w_qkvu;         /* [4d][d] (dtype) */
  const void* w1;             /* [d_ff][d] (dtype) */
  const void* w2;             /* [d][d_ff] (dtype) */
  const float* b_qkvu;        /* [4d] or NULL */
  const float* b1;            /* [d_ff] or NULL */
  const float* b2;            /* [d] or NULL */
  const float* rab_pos;       /* MTGR_VARIANT_RAB: [H][2 MTGR_RAB_MAX_DIST + 1], else unused */
  const float* rab_time;      /* MTGR_VARIANT_RAB: [H][MTGR_RAB_TIME_BUCKETS], else unused */
} mtgr_block_params;

/* Workspace bytes of mtgr_hstu_block_fwd for T tokens (0 on invalid params). */
MTGR_API size_t mtgr_block_workspace_bytes(int32_t T, const mtgr_block_params* p);

/*
 * One HSTU block (summary page, Method, the update equations). The residual
 * stream is float32 on both paths: d_x_in, d_x_out [T][d] float32 (distinct
 * buffers). dtype MTGR_BF16: GroupLN outputs and GEMM operands in bf16,
 * Q|K|V|U and the attention probabilities in fp16, fp32 accumulation
 * (d % 64 == 0, dh == 64, d_ff % 64 == 0). dtype MTGR_F32: every step in fp32
 * on CUDA cores (dh in {32, 64}).
 */
MTGR_API int mtgr_hstu_block_fwd(const mtgr_block_params* p, const mtgr_batch* batch,
                                 const float* d_x_in, float* d_x_out, void* d_ws,
                                 size_t ws_bytes, mtgr_stream_t stream);

/* Workspace bytes of mtgr_stack_fwd (0 on invalid params). */
MTGR_API size_t mtgr_stack_workspace_bytes(int32_t T, const mtgr_block_params* layers, int32_t L);

/*
 * L stacked HSTU blocks (summary page, Method: the L-layer stack). The mask
 * metadata in *batch is shared by all layers. d_x_in and d_x_out [T][d]
 * float32, distinct. All layers must share d, H and dtype.
 */
MTGR_API int mtgr_stack_fwd(const mtgr_block_params* layers, int32_t L, const mtgr_batch* batch,
                            const float* d_x_in, float* d_x_out, void* d_ws, size_t ws_bytes,
                            mtgr_stream_t stream);

/*
 * The whole forward from HOST buffers, for callers that keep their batches in
 * host memory (a C serving process, or a pipeline that stages batches from
 * disk): one call enqueues on `stream` the copies of the lengths, timestamps,
 * optional normalisers and token features into the device workspace, the
 * packing, the mask metadata, the L-block stack and the copies of the output
 * rows and the status word back to the host. Nothing is allocated: the device
 * workspace (mtgr_stack_fwd_host_workspace_bytes) holds the staged inputs,
 * the batch, its metadata and the stack's workspace.
 *   h_lens [B][4] int32, h_ts [T] int64, h_norm [B] float (or NULL),
 *   h_x_in, h_x_out [T][d] float32: HOST memory, pinned (page-locked) for the
 *     copies to be asynchronous; they must stay valid and untouched until
 *     the stream has passed this call's work
 *   h_status: host int32, written by the final copy (0 = ok, else a device
 *     status such as MTGR_ERR_DEVICE_VALIDATION), valid once the stream has
 *     synchronised
 * T is the sum of h_lens (computed here, on the host). Calls sharing a
 * workspace must be ordered; two workspaces on two streams let one call's
 * copies overlap the other's kernels.
 */
MTGR_API size_t mtgr_stack_fwd_host_workspace_bytes(int32_t B, const int32_t* h_lens,
                                                    const mtgr_block_params* layers, int32_t L);
MTGR_API int mtgr_stack_fwd_host(const mtgr_block_params* layers, int32_t L, int32_t B,
                                 const int32_t* h_lens, const int64_t* h_ts, const float* h_norm,
                                 const float* h_x_in, float* h_x_out, int32_t* h_status,
                                 void* d_ws, size_t ws_bytes, mtgr_stream_t stream);

/*
 * Candidate-incremental scoring (serving). A user's U, S and R tokens never
 * attend to candidates (mask rules 1-3), so the context side of every layer
 * is computed once and candidates are scored against it afterwards, in one
 * or more chunks (fun-rec 7.3.4: at inference the candidates of a request
 * are independent of one another; the MTGR practice article, 5.2 on
 * inference latency: cache the User/Seq tokens, which change rarely).
 *
 * mtgr_restrict_work: rewrites batch->work and counts[3] in place so that
 * the attention computes only the work items holding a query row at or
 * after d_q_first[b] (user-relative, int32 [B], device; NULL: each user's
 * first candidate row N_U + N_S + N_R); a q-tile pair whose first q-tile
 * lies wholly before it becomes a single-q-tile item. Order is kept;
 * restricting twice to the same rows changes nothing. Call after
 * mtgr_build_mask_meta on the same stream.
 */
MTGR_API int mtgr_restrict_work(const mtgr_batch* batch, const int32_t* d_q_first,
                                mtgr_stream_t stream);

/* Workspace bytes of mtgr_stack_fwd_rows (0 on invalid params; bf16 only). */
MTGR_API size_t mtgr_stack_rows_workspace_bytes(int32_t T, int32_t row0,
                                                const mtgr_block_params* layers, int32_t L);

/*
 * L bf16 blocks on rows [row0, T) of the batch, with every layer's Q|K|V|U
 * kept in a caller-owned cache: layer l uses rows [0, T) of
 * d_qkvu_cache + l * cache_rows * 4d (f16, [cache_rows][4d] per layer,
 * cache_rows >= T, Q columns halved). Rows [row0, T) of each layer's slot
 * are written; rows before row0 must already hold that layer's Q|K|V|U.
 * d_x_in, d_x_out: [T - row0][d] float32, distinct.
 *   Context pass: the user's U, S, R tokens as the batch (lens (N_U, N_S,
 *     N_R, 0), normaliser override N = N_U + N_S + N_R + K for the K
 *     candidates to come), row0 = 0.
 *   Candidate pass: one user (B = 1) holding the same U, S, R tokens and a
 *     chunk of candidates (lens (N_U, N_S, N_R, k), same timestamps and
 *     normaliser N), row0 = N_U + N_S + N_R, work list restricted with
 *     mtgr_restrict_work to rows >= row0; writes the k candidates' outputs.
 *     Rows [row0, T) of the cache are overwritten, so chunks run one after
 *     another. The result equals the candidate rows of the aggregated pass
 *     over [U, S, R, all candidates] with the same N, up to the rounding
 *     order of each candidate's self term.
 */
MTGR_API int mtgr_stack_fwd_rows(const mtgr_block_params* layers, int32_t L,
                                 const mtgr_batch* batch, int32_t row0, void* d_qkvu_cache,
                                 int32_t cache_rows, const float* d_x_in, float* d_x_out,
                                 void* d_ws, size_t ws_bytes, mtgr_stream_t stream);

/*
 * Token MLPs and candidate heads: the steps on either side of the stack
 * (blog posts "generative recommendation 18: MTGR", "Converting
 * heterogeneous features into tokens"; summary page, "Method"; fun-rec
 * 7.3.3: CandidateToken_i = MLP(Concat(Emb(Item_i), Emb(Cross_i)))).
 *
 * One domain's token MLP: Linear(f, d) -> SiLU -> Linear(d, d).
 */
typedef struct mtgr_token_mlp {
  int32_t f;          /* input width (concatenated field embeddings), % 64 == 0 */
  int32_t reserved;
  const void* w1;     /* [d][f] bf16 */
  const float* b1;    /* [d] or NULL */
  const void* w2;     /* [d][d] bf16 */
  const float* b2;    /* [d] or NULL */
} mtgr_token_mlp;

/* Workspace bytes of mtgr_tokenize (0 on invalid sizes). */
MTGR_API size_t mtgr_tokenize_workspace_bytes(int32_t B, int32_t d, const int32_t n_rows[4]);

/*
 * Builds the block input X of a packed batch from per-domain inputs:
 *   d_e[0]: U tokens, bf16 [n_rows[0]][d] (the feature embeddings; no MLP);
 *   d_e[g], g = 1, 2, 3 (S, R, C): bf16 [n_rows[g]][mlp[g-1].f], the
 *     concatenated field embeddings, through mlp[g-1].
 * Each input lists its domain's tokens user by user, each user's in sequence
 * order; X row seg_off[4b + g] + j (float32 [T][d]) gets user b's j-th token
 * of domain g. n_rows (host) must equal the batch's per-domain totals; a
 * mismatch is a device error (MTGR_ERR_DEVICE_VALIDATION in the batch status)
 * and X is then undefined. d % 64 == 0; all pointers 16-byte aligned.
 */
MTGR_API int mtgr_tokenize(const mtgr_batch* batch, int32_t d, const int32_t n_rows[4],
                           const void* const d_e[4], const mtgr_token_mlp mlp[3], float* d_x,
                           void* d_ws, size_t ws_bytes, mtgr_stream_t stream);

/* Task heads on the candidates' rows: per task t, Linear(d, d_h) -> SiLU ->
 * Linear(d_h, 1), giving a logit (CTR, CTCVR, ...). */
typedef struct mtgr_head_params {
  int32_t d;          /* d_model, % 64 == 0 */
  int32_t d_h;        /* hidden width per task, % 32 == 0 */
  int32_t n_tasks;    /* >= 1 */
  int32_t reserved;
  const void* w1;     /* [n_tasks * d_h][d] bf16 (task t: rows [t d_h, (t+1) d_h)) */
  const float* b1;    /* [n_tasks * d_h] or NULL */
  const float* w2;    /* [n_tasks][d_h] float32 */
  const float* b2;    /* [n_tasks] or NULL */
} mtgr_head_params;

/* Workspace bytes of mtgr_candidate_heads (0 on invalid params). */
MTGR_API size_t mtgr_heads_workspace_bytes(int32_t B, int32_t k_total, const mtgr_head_params* p);

/*
 * Logits d_out float32 [k_total][n_tasks] of the candidates of the batch,
 * user by user, each user's in sequence order, from its output rows d_x
 * float32 [T][d]. k_total (host) must equal the batch's candidate count; a
 * mismatch is a device error as for mtgr_tokenize.
 */
MTGR_API int mtgr_candidate_heads(const mtgr_head_params* p, const mtgr_batch* batch,
                                  int32_t k_total, const float* d_x, float* d_out, void* d_ws,
                                  size_t ws_bytes, mtgr_stream_t stream);

/*
 * Cached-context candidate pass over a whole batch of users.
 *   Context pass (once per set of contexts): mtgr_stack_fwd_rows with
 *     row0 = 0 over a batch with lens (N_U, N_S, N_R, K_b) per user, the
 *     candidate rows holding anything (zeros), with the normaliser override
 *     N_b = N_U + N_S + N_R + K_b. A context row never sees a candidate, so
 *     every layer's Q|K|V|U of the context rows is final.
 *   Candidate pass: a batch of the same lens with the real candidates'
 *     timestamps (same normalisers), and mtgr_stack_fwd_candidates: every
 *     layer computes the candidate rows only. Their Q|K|V|U go into the
 *     cache at their packed rows, the attention runs over the candidates'
 *     q-tiles, and GroupLN and the MLP run on the candidates' rows.
 * d_x_cand, d_x_out: float32 [k_total][d], the candidates user by user
 * (k_total = sum K_b, checked on the device: MTGR_ERR_DEVICE_VALIDATION in
 * the batch status). d_qkvu_cache as for mtgr_stack_fwd_rows
 * (cache_rows >= T). The batch's work list is restricted in place to the
 * candidates' q-tiles. Candidate rows sit where the aggregated pass has them,
 * so the result equals that pass's candidate rows. Not with
 * MTGR_VARIANT_POOLED_GLN (MTGR_ERR_UNSUPPORTED).
 */
MTGR_API size_t mtgr_stack_candidates_workspace_bytes(int32_t B, int32_t T, int32_t k_total,
                                                      const mtgr_block_params* layers, int32_t L);
MTGR_API int mtgr_stack_fwd_candidates(const mtgr_block_params* layers, int32_t L,
                                       const mtgr_batch* batch, int32_t k_total, void* d_qkvu_cache,
                                       int32_t cache_rows, const float* d_x_cand, float* d_x_out,
                                       void* d_ws, size_t ws_bytes, mtgr_stream_t stream);

/*
 * Dense GEMM with the block's epilogues, exposed for testing:
 *   out[m][n] = epi( sum_k a[m][k] * b[n][k] + bias[n] )
 *   epi = MTGR_EPI_NONE (out dtype MTGR_F16/MTGR_BF16/MTGR_F32),
 *         MTGR_EPI_SILU (out MTGR_F16/MTGR_BF16/MTGR_F32),
 *         MTGR_EPI_RESID (adds d_resid[m][n] float32; out MTGR_F32)
 *   ab_dtype MTGR_BF16: tcgen05 tensor cores (K % 64 == 0, N % 32 == 0);
 *   ab_dtype MTGR_F32: CUDA cores. a [M][K], b [N][K] row-major; bias may
 *   be NULL. q_cols > 0 multiplies output columns [0, q_cols) by 0.5 after
 *   the SiLU and before the conversion (used to pre-halve Q for the attention).
 */
#define MTGR_EPI_NONE 0
#define MTGR_EPI_SILU 1
#define MTGR_EPI_RESID 2
MTGR_API int mtgr_gemm(int32_t M, int32_t N, int32_t K, int32_t ab_dtype, const void* d_a,
                       const void* d_b, const float* d_bias, int32_t epi, const float* d_resid,
                       int32_t q_cols, int32_t out_dtype, void* d_out, int32_t* d_status,
                       mtgr_stream_t stream);

/*
 * Weight-gradient GEMM of the block's backward, exposed for testing: the
 * gradient of a Linear layer's weight is a sum over tokens of two activation
 * rows (summary page, "Method": the block's projections, their gradients by
 * the chain rule),
 *   out[m][n] (+)= sum_t a[t][m] * b[t][n]
 * a [T][lda] and b [T][ldb] bf16, token-major as the forward wrote them
 * (the first M, resp. N, values of each row are used); out [M][N] fp32,
 * row-major. accumulate == 0 zeroes out first; otherwise the sums are added
 * to what it holds. Runs on tcgen05 CTA pairs with fp32 reduce-add of
 * partial tiles, so the summation order over tokens varies from run to run
 * (results agree to fp32 rounding). lda, ldb: multiples of 8 elements, at
 * least M, N; N a multiple of 4; pointers 16-byte aligned. The caller owns
 * every buffer. Returns MTGR_ERR_INVALID_ARG for a bad size, stride,
 * alignment or a NULL pointer, MTGR_ERR_UNSUPPORTED off sm_100;
 * MTGR_ERR_TIMEOUT is written to d_status if a wait inside the kernel runs
 * out. Timer class MTGR_TIMER_BWD_WGRAD.
 */
MTGR_API int mtgr_gemm_wgrad(int32_t M, int32_t N, int64_t T, const void* d_a, int64_t lda,
                             const void* d_b, int64_t ldb, float* d_out, int32_t accumulate,
                             int32_t* d_status, mtgr_stream_t stream);

/*
 * Kernel timing. A timer attached to the calling host thread makes every
 * entry point bracket its kernels with CUDA events on its stream and count
 * them, per class: MTGR_TIMER_PACK (2 kernels per call), MTGR_TIMER_MASK_META
 * (6), MTGR_TIMER_GLN, MTGR_TIMER_GEMM_QKVU, MTGR_TIMER_ATTENTION,
 * MTGR_TIMER_GEMM_MLP1, MTGR_TIMER_GEMM_MLP2 (1 each; mtgr_gemm counts as
 * MTGR_TIMER_GEMM_QKVU); MTGR_TIMER_TOKEN_MLP (the token MLPs' GEMMs, 2 per
 * domain with tokens), MTGR_TIMER_HEAD_MLP (the heads' first layer, 1) and
 * MTGR_TIMER_ROWS (the row bookkeeping of tokenize, heads and the candidate
 * pass: 3, 4, and 3 + 1 per layer). mtgr_timer_read synchronises on the recorded events,
 * writes the summed milliseconds and launch counts per class into
 * ms[MTGR_TIMER_CLASSES] and launches[MTGR_TIMER_CLASSES] (host arrays) and
 * clears the records. Attaching NULL detaches. Not for use during CUDA graph
 * capture.
 */
#define MTGR_TIMER_PACK 0
#define MTGR_TIMER_MASK_META 1
#define MTGR_TIMER_GLN 2
#define MTGR_TIMER_GEMM_QKVU 3
#define MTGR_TIMER_ATTENTION 4
#define MTGR_TIMER_GEMM_MLP1 5
#define MTGR_TIMER_GEMM_MLP2 6
#define MTGR_TIMER_TOKEN_MLP 7
#define MTGR_TIMER_HEAD_MLP 8
#define MTGR_TIMER_ROWS 9
#define MTGR_TIMER_BWD_GEMM 10      /* backward: dH, dG~, dX~ GEMMs (3 per block) */
#define MTGR_TIMER_BWD_WGRAD 11     /* backward: dW2, dW1, dW_qkvu GEMMs (3) */
#define MTGR_TIMER_BWD_ATTENTION 12 /* backward: attention (1, plus its k-tile list) */
#define MTGR_TIMER_BWD_GLN 13       /* backward: both GroupLNs (2) */
#define MTGR_TIMER_BWD_ROWS 14      /* backward: conversions, transposes, column sums */
#define MTGR_TIMER_CLASSES 15
typedef struct mtgr_timer mtgr_timer;
MTGR_API mtgr_timer* mtgr_timer_create(void);
MTGR_API void mtgr_timer_destroy(mtgr_timer* timer);
MTGR_API int mtgr_timer_attach(mtgr_timer* timer);
MTGR_API int mtgr_timer_read(mtgr_timer* timer, double* ms, int64_t* launches);

/*
 * Training: the block's forward keeping what its backward reads, and the
 * backward (the gradients of the summary page's Method update equations by
 * the chain rule; the pages' system numbers are training throughput, in
 * bf16 mixed precision: summary page, main contributions and Method, the
 * training system). Variant 0 blocks only (MTGR_ERR_UNSUPPORTED otherwise).
 *
 * mtgr_hstu_block_fwd_train: as mtgr_hstu_block_fwd, and d_saved (caller
 * owned, mtgr_block_saved_bytes(T, p) bytes) receives the activations the
 * backward reads: GroupLN_1 output, Q|K|V|U, O/N (the attention before the
 * gate), G, GroupLN_2 output, the MLP pre-activation and its SiLU (bf16
 * blocks: bf16, Q|K|V|U f16 with Q halved; fp32 blocks: fp32). Same output
 * x_out as mtgr_hstu_block_fwd.
 */
MTGR_API size_t mtgr_block_saved_bytes(int32_t T, const mtgr_block_params* p);
MTGR_API int mtgr_hstu_block_fwd_train(const mtgr_block_params* p, const mtgr_batch* batch,
                                       const float* d_x_in, float* d_x_out, void* d_saved,
                                       size_t saved_bytes, mtgr_stream_t stream);

/* Parameter gradients of one block (device, fp32, same shapes as the
 * parameters; written, not accumulated). A NULL bias entry skips that bias's
 * gradient; every other entry is required. */
typedef struct mtgr_block_grads {
  float* gln1_gamma;  /* [4][d] */
  float* gln1_beta;   /* [4][d] */
  float* w_qkvu;      /* [4d][d] */
  float* b_qkvu;      /* [4d] or NULL */
  float* gln2_gamma;  /* [4][d] */
  float* gln2_beta;   /* [4][d] */
  float* w1;          /* [d_ff][d] */
  float* b1;          /* [d_ff] or NULL */
  float* w2;          /* [d][d_ff] */
  float* b2;          /* [d] or NULL */
} mtgr_block_grads;

/*
 * Backward of one block: given d_dy = dL/dX_out [T][d] fp32, writes
 * d_dx = dL/dX_in [T][d] fp32 and the parameter gradients. d_x_in and
 * d_saved are the forward's input and saved activations (same batch,
 * parameters and normaliser). Workspace: mtgr_block_bwd_workspace_bytes.
 * bf16 blocks run the contractions on tcgen05 tensor cores (the attention's
 * with f16 operands, its dO~ = dG (.) U in f16: values beyond 65504 set
 * MTGR_ERR_RANGE in the batch status, values below 2^-14 lose precision as
 * f16 subnormals, so scale the loss as usual for f16 training), and keep the
 * gradients of the GroupLN outputs (dG~, dX~) in bf16 between a GEMM and the
 * GroupLN backward that reads them; fp32 blocks run on CUDA cores in fp32
 * throughout. Weight gradients are sums over all tokens accumulated in fp32
 * in an order that varies from run to run.
 */
MTGR_API size_t mtgr_block_bwd_workspace_bytes(int32_t T, const mtgr_block_params* p,
                                               const mtgr_batch* batch);
MTGR_API int mtgr_hstu_block_bwd(const mtgr_block_params* p, const mtgr_batch* batch,
                                 const float* d_x_in, const void* d_saved, const float* d_dy,
                                 float* d_dx, const mtgr_block_grads* grads, void* d_ws,
                                 size_t ws_bytes, mtgr_stream_t stream);

/*
 * Self-test of the bounded waits (failure handling, not part of the method):
 * every internal wait of the library's tensor-core kernels gives up after a
 * limit, records MTGR_ERR_TIMEOUT in the caller's status word, frees the
 * kernel's tensor memory and returns, so that a protocol fault can never hang
 * the GPU. This entry point launches one block of that shape whose waits can
 * never be satisfied, under the given limit, so the whole wind-down runs:
 * after the stream is synchronised, *d_status holds MTGR_ERR_TIMEOUT (if it
 * was 0) and the device stays usable for the next launch.
 *   limit_ns  per-wait limit in nanoseconds, 1e3 <= limit_ns <= 1e9
 *             (MTGR_ERR_INVALID_ARG otherwise)
 *   d_status  device int32 status word
 */
MTGR_API int mtgr_selftest_bounded_wait(uint64_t limit_ns, int32_t* d_status,
                                        mtgr_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MTGR_H */
