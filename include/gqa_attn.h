/*
 * gqa_attn.h -- C ABI of the B200 (sm_100a) exact grouped-query attention forward.
 *
 * Operation (every entry point computes the same definition):
 *   for each batch element (or packed sequence) b and query head h, with
 *   G = Hq / Hkv and key/value head c = h / G,
 *     S[i, j] = scale * sum_d q[b, i, h, d] * k[b, j, c, d]
 *     S[i, j] = -inf where causal and j > i + (Sk - Sq)
 *     O[b, i, h, :] = sum_j softmax_j(S[i, :]) v[b, j, c, :]
 *     L[b, h, i]    = ln sum_j exp(S[i, j])
 *   Sources: FlashAttention-2 summary page (azimuth.plus) -- standard attention
 *   S = QK^T, P = softmax(S), O = PV; tiled online softmax with running max m
 *   and sum l, deferred normalisation, L = m + log l; causal mask (entries above
 *   the diagonal are -inf, the diagonal is kept).  Ultralytics glossary
 *   "Grouped Query Attention (GQA)", section "How GQA works" -- groups of Hq/Hkv
 *   query heads share one K/V head; Hkv = 1 is MQA and Hkv = Hq is MHA.
 *   Interface shape: flash_attn_func(q, k, v, dropout_p, softmax_scale, causal)
 *   on [batch, seq_len, num_heads, head_dim] tensors (StructBERT/FlashAttention
 *   page, section 2.2) and flash_attn_func(q, k, v, pack_gqa=..., num_splits=...)
 *   (GQA batch-size guide, "Dynamic parameter tuning").
 *   Readings where the pages are silent: causal masks are bottom-right aligned
 *   when Sq != Sk (a single decode query sees every key); a row with no visible
 *   key gets O = 0 and L = -inf; L is the natural log of the scaled logits.
 *
 * Memory and layout:
 *   All tensor pointers are DEVICE pointers owned by the caller; the library
 *   never allocates, frees or synchronises.  Every call is enqueued on `stream`
 *   and returns after the enqueue (stream-ordered, no host sync inside), so a
 *   call may be captured in a CUDA graph once its workspace is registered.
 *   Dense:  q, out [B, Sq, Hq, D]; k, v [B, Sk, Hkv, D]; lse [B, Hq, Sq] fp32;
 *           all contiguous row-major.
 *   Packed variable-length (cu_seqlens != NULL): q, out [total, Hq, D];
 *           k, v [total, Hkv, D]; lse [Hq, total]; cu_seqlens is a device int32
 *           array [B + 1], non-decreasing, cu_seqlens[0] = 0, cu_seqlens[B] =
 *           total; sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1 of q,
 *           k and v (self-attention: its query and key lengths are its length).
 *           The caller passes Sq = the largest sequence length (an upper bound
 *           is accepted) and Sk = total, the number of packed rows it allocated:
 *           TMA descriptors are sized from it, so nothing past the buffers is
 *           read.  A sequence longer than Sq, or cu_seqlens[B] > Sk, raises
 *           device error 2 and the offending tiles are not trusted.
 *   Tensor pointers must be 16-byte aligned (TMA), lse 4-byte aligned.
 *
 * Errors: every entry point returns a gqa_status (0 = success).  Argument errors
 *   are detected on the host before anything is enqueued.  GQA_ERR_CUDA reports
 *   a failed launch (cudaGetLastError).  Kernels never trap: a pipeline wait that
 *   exceeds its time limit records a device error code and the kernel returns;
 *   read it with gqa_attn_get_device_error().
 */
#ifndef GQA_ATTN_H
#define GQA_ATTN_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GQA_OK = 0,
    GQA_ERR_NULL = -1,        /* a required pointer is NULL */
    GQA_ERR_SHAPE = -2,       /* negative sizes, Hq % Hkv != 0, index range overflow */
    GQA_ERR_HEADDIM = -3,     /* D not supported (bf16: 64 or 128; fp32: 1..256) */
    GQA_ERR_ALIGN = -4,       /* tensor pointer not 16-byte aligned (lse: 4-byte) */
    GQA_ERR_SPLITS = -5,      /* num_splits < 0, > 256, or > 1 outside dense Sq == 1 */
    GQA_ERR_WORKSPACE = -6,   /* num_splits > 1 and the registered workspace is too small */
    GQA_ERR_SCALE = -7,       /* scale not finite or not > 0 */
    GQA_ERR_CUDA = -8,        /* a CUDA runtime call or a launch failed */
    GQA_ERR_UNSUPPORTED = -9  /* device is not sm_100, or pack_gqa not in {-1, 0, 1} */
} gqa_status;

/*
 * bf16 forward (fp32 accumulation, bf16 output, fp32 lse).
 *   q, k, v, out : bf16 tensors as described above
 *   lse          : fp32 log-sum-exp per (b, h, query row)
 *   B            : batch size, or number of packed sequences when cu_seqlens != NULL
 *   Hq, Hkv      : query heads and key/value heads (Hq % Hkv == 0)
 *   Sq, Sk       : query and key lengths (varlen: Sq = maximum length,
 *                  Sk = total packed rows)
 *   D            : head dimension, 64 or 128
 *   scale        : softmax scale (finite, > 0); 1/sqrt(D) is the usual choice
 *   causal       : nonzero for the causal mask
 *   num_splits   : split-KV factor for decode (dense, Sq == 1): 1 = none,
 *                  n > 1 = n contiguous key ranges combined by log-sum-exp
 *                  (needs a workspace, see below), 0 = chosen by the library
 *                  (as many splits as give every CTA an SM of its own).  With
 *                  n > 1 two kernels are enqueued: the split kernel and the
 *                  combine, the latter as a programmatic dependent launch.
 *                  Must be 0 or 1 for every other shape.
 *   pack_gqa     : 1 = the G query heads of a KV head share one tile (K/V read
 *                  once per group), 0 = one query head per tile, -1 = chosen by
 *                  the library.  Changes speed only, never the definition.
 *   cu_seqlens   : NULL (dense) or device int32[B + 1] (packed variable length)
 *   stream       : CUDA stream the work is enqueued on
 */
int gqa_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                 int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                 int num_splits, int pack_gqa, const int* cu_seqlens, cudaStream_t stream);

/*
 * fp32 forward: same parameters and layouts with fp32 q, k, v and out, computed
 * in fp32 on CUDA cores.  D may be 1..256; num_splits must be 0 or 1; pack_gqa
 * is accepted and ignored.
 */
int gqa_attn_fwd_f32(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                     int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                     int num_splits, int pack_gqa, const int* cu_seqlens, cudaStream_t stream);

/*
 * gqa_attn_fwd on inputs and outputs in host memory, with the transfers overlapped:
 * the problem is cut into `chunks` pieces (0 = 8; at most 64) and, on three streams the
 * library creates once per device, the copy of piece c+1 to the device, the attention
 * of piece c and the copy of piece c-1's results back run at the same time.  Pieces are
 * groups of whole batch elements; when the batch has fewer elements than `chunks`, a
 * prefill (Sq >= 512; causal only with Sq <= Sk) is cut into ranges of query positions
 * of each batch element instead, each copying in the keys its queries newly see (the
 * results are those of gqa_attn_fwd, bit for bit).  Dense only (no cu_seqlens), bf16.
 *   q_h, k_h, v_h, out_h, lse_h : host buffers in gqa_attn_fwd's layouts; page-locked
 *                  (cudaHostAlloc / cudaHostRegister) for the copies to overlap
 *   q_d ... lse_d : caller-owned device buffers of the same sizes (the staging area;
 *                  they hold the inputs and results afterwards)
 *   other arguments as gqa_attn_fwd; a split-KV decode chunk uses the workspace
 *                  registered for the current device, sized for its own batch
 * Ordered after earlier work on `stream`; later work on `stream` waits for all of it.
 * One call at a time per device from the library's side (calls from several host
 * threads are serialised while they enqueue).  Returns gqa_attn_fwd's status codes;
 * GQA_ERR_SHAPE also for chunks < 0 or > 64.  This entry point has no counterpart
 * on the pages: it exists so that host-resident inputs reach the kernels with the
 * transfers hidden behind the computation.
 */
int gqa_attn_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* out_h,
                      float* lse_h, void* q_d, void* k_d, void* v_d, void* out_d, float* lse_d,
                      int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                      int num_splits, int pack_gqa, int chunks, cudaStream_t stream);

/*
 * The packed variable-length form of gqa_attn_fwd_host: chunks of whole sequences
 * (about total / chunks rows each; 0 = 8 chunks) are copied in, computed and copied
 * back with the same overlap.
 *   q_h .. lse_h : host buffers, packed layouts of gqa_attn_fwd (q/out [total, Hq, D],
 *                  k/v [total, Hkv, D], lse [Hq, total]); page-locked for overlap
 *   q_d .. lse_d : device buffers of the same sizes
 *   cu_seqlens_h : host int32[B + 1] (0 = cu[0] <= ... <= cu[B] = total), used to cut
 *                  the chunks; cu_seqlens_d: the same offsets in device memory, read by
 *                  the kernels
 *   max_seqlen   : the longest sequence; total: packed rows
 * Returns gqa_attn_fwd's status codes; GQA_ERR_SHAPE also when cu_seqlens_h does not
 * describe `total` rows with no sequence longer than max_seqlen, or for chunks < 0 or
 * > 64.  No counterpart on the pages (see gqa_attn_fwd_host).
 */
int gqa_attn_fwd_host_varlen(const void* q_h, const void* k_h, const void* v_h, void* out_h,
                             float* lse_h, void* q_d, void* k_d, void* v_d, void* out_d,
                             float* lse_d, const int* cu_seqlens_h, const int* cu_seqlens_d,
                             int B, int Hq, int Hkv, int max_seqlen, int total, int D,
                             float scale, int causal, int pack_gqa, int chunks,
                             cudaStream_t stream);

/*
 * Bytes of device workspace gqa_attn_fwd needs for a split-KV decode with the
 * given sizes and num_splits (0 when num_splits <= 1): fp32 partial outputs
 * [B, Hq, Sq, n, D] and partial log-sum-exps [B, Hq, Sq, n].
 */
size_t gqa_attn_workspace_bytes(int B, int Hq, int Sq, int D, int num_splits);

/*
 * Register a caller-owned device buffer as the split-KV workspace of the calling
 * thread's current device (one registration per device and process; borrowed,
 * never freed by the library; NULL/0 unregisters).  Calls that run concurrently
 * on different streams must not share one workspace.  Returns GQA_ERR_ALIGN if
 * dev_ptr is not 16-byte aligned, GQA_ERR_CUDA if no device can be queried.
 */
int gqa_attn_set_workspace(void* dev_ptr, size_t bytes);

/*
 * The choices gqa_attn_fwd makes for these arguments, without launching:
 *   *kernel = 0 nothing to do, 1 sm_100a tcgen05 prefill, 2 split-KV decode,
 *             3 zero fill (no keys);
 *   *splits and *pack = the effective num_splits and pack_gqa.
 * Returns the status gqa_attn_fwd would return for the argument checks that do
 * not need pointers (shape, head dim, splits, pack, scale, device).
 */
int gqa_attn_plan(int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                  int num_splits, int pack_gqa, int varlen, int* kernel, int* splits,
                  int* pack);

/*
 * Read and clear the device error word on `stream` (synchronises that stream).
 * *host_code: 0 none, 1 a pipeline wait timed out, 2 a packed sequence is longer
 * than the Sq that was passed, 3 a KV-cache length or page index outside the cache.
 */
int gqa_attn_get_device_error(int* host_code, cudaStream_t stream);

/*
 * Split-KV decode that allocates nothing (no counterpart on the pages; it is an
 * addition for callers that cannot obtain device memory at call time).
 *
 * Who needs it: code that runs where allocation is unavailable or forbidden --
 * a plugin or custom op handed only its input and output buffers by a host
 * engine that owns all memory, a real-time loop whose latency budget cannot absorb
 * cudaMalloc (which may synchronise the device), or a caller with no allocator of
 * its own.  gqa_attn_fwd's split-KV path needs a workspace registered beforehand;
 * this entry point needs none: its partial results go to a scratch array of
 * GQA_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU that loads
 * the library keeps for the life of the process.
 *
 * Computes exactly what gqa_attn_fwd computes for a dense decode step (Sq = 1,
 * causal or not: one query sees every key) with the same q [B,1,Hq,D], k/v
 * [B,Sk,Hkv,D], out and lse [B,Hq,1] layouts, bf16 in/out, D 64 or 128, and the
 * same num_splits (0 = automatic, reduced until the partials fit the scratch) and
 * pack_gqa meanings.  Nothing is allocated, freed or synchronised: no cudaMalloc,
 * no cudaFree, no allocating library call.
 *
 * Limits and sharing:
 *   - B * Hq * num_splits * (D + 1) * 4 bytes (plus alignment) must fit in
 *     GQA_NOALLOC_SCRATCH_BYTES; an explicit num_splits that does not fit returns
 *     GQA_ERR_WORKSPACE and launches nothing;
 *   - every call in the process shares the one array per device and leaves its
 *     partials there; the next call overwrites them (each partial is written
 *     before it is read within a call, so nothing needs clearing), but calls that
 *     overlap on the GPU (different streams, or concurrent host threads) race on
 *     it and must be serialised by the caller;
 *   - the first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 * Returns the same status codes as gqa_attn_fwd.
 */
#define GQA_NOALLOC_SCRATCH_BYTES (4u << 20)
int gqa_attn_decode_noalloc(const void* q, const void* k, const void* v, void* out,
                            float* lse, int B, int Hq, int Hkv, int Sk, int D, float scale,
                            int num_splits, int pack_gqa, cudaStream_t stream);

/*
 * Backward pass of the dense forward: dQ, dK, dV for a given dO (FA-2 summary page,
 * backward paragraph: dK and dV accumulate per K/V column block, dQ is shared between
 * them; GQA paragraph: dK and dV are summed over the query heads sharing a K/V head).
 * With P recomputed from lse and D_i = rowsum(dO_i * O_i):
 *   dV = P^T dO;  dS = P * (dO V^T - D);  dK = scale dS^T Q;  dQ = scale dS K.
 * q, out, dout, dq [B, Sq, Hq, D]; k, v, dk, dv [B, Sk, Hkv, D] (bf16, contiguous);
 * lse [B, Hq, Sq] fp32 as gqa_attn_fwd wrote it with the same q, k, v, scale and
 * causal; D 64 or 128; causal as gqa_attn_fwd (bottom-right).  Every output element is
 * written (no accumulation into the caller's buffers, no atomics: run to run the
 * results are bit-identical).  The registered workspace (gqa_attn_set_workspace) must
 * hold gqa_attn_bwd_workspace_bytes(B, Hq, Sq) bytes (GQA_ERR_WORKSPACE otherwise);
 * nothing is allocated or synchronised.  Status codes as gqa_attn_fwd.
 */
size_t gqa_attn_bwd_workspace_bytes(int B, int Hq, int Sq);
int gqa_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq,
                 int Sk, int D, float scale, int causal, cudaStream_t stream);

/*
 * Block-sparse attention: gqa_attn_fwd's dense forward restricted to a pattern of
 * (query block, key block) pairs with blocks of 128 positions and 128 keys (Raptor-T
 * abstract: BigBird divides the input into blocks of a block size and computes
 * attention between blocks, several patterns combined into one).
 *   key j is visible to query i iff j / 128 is in row i / 128 of the pattern and, when
 *   causal != 0, j <= i + (Sk - Sq) as well (gqa_attn_fwd's causal mask);
 *   blk_row_ptr: device int32 [ceil(Sq / 128) + 1], blk_row_ptr[0] = 0, non-
 *     decreasing; blk_col: device int32 [blk_row_ptr[last]], the key blocks of each
 *     row, in [0, ceil(Sk / 128)) (an entry outside raises device error 2 and block 0
 *     is read in its place), ascending within a row (any order gives the same result);
 *   the pattern is the same for every batch element and head;
 *   a query whose blocks hold no key gets O = 0, L = -inf.
 * Layouts, dtypes (bf16 only), D (64, 128) and errors as gqa_attn_fwd.  PackGQA is
 * always on, and the group size G = Hq / Hkv must be >= 2 and divide 128 (one CTA tile
 * of 256 / G positions then lies in one query block); otherwise GQA_ERR_UNSUPPORTED.
 */
int gqa_attn_fwd_blocksparse(const void* q, const void* k, const void* v, void* out, float* lse,
                             int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                             int causal, const int* blk_row_ptr, const int* blk_col,
                             cudaStream_t stream);

/*
 * Causal forward within a sliding window (Ultralytics glossary, "GQA and related
 * techniques": sliding-window attention caps the tokens each token attends to, paired
 * there with GQA).  Reading taken where the page gives no formula: query i, at key
 * position i + (Sk - Sq), sees its `window` most recent keys,
 *   key j visible to query i iff i + (Sk - Sq) - window < j <= i + (Sk - Sq),
 * the same window as the decode entry points' (the newest query sees the last
 * `window` keys).  window >= 1 (GQA_ERR_SHAPE otherwise); a window holding every key
 * is gqa_attn_fwd with causal = 1.  Arguments, layouts (dense or packed with
 * cu_seqlens), dtypes (bf16), D, pack_gqa and errors as gqa_attn_fwd; one query
 * (Sq = 1, dense) runs the decode kernel without splits.
 */
int gqa_attn_fwd_window(const void* q, const void* k, const void* v, void* out, float* lse,
                        int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int window,
                        int pack_gqa, const int* cu_seqlens, cudaStream_t stream);

/*
 * Prefill forward on e4m3 Q, K and V with one scale per tensor (the batch-size guide
 * names FP8 as the precision that lowers memory-bandwidth pressure: hardware adaptation
 * section, Hopper item; precision row of its production checklist).
 *   element = value(code) * scale of its tensor; q8 [B, Sq, Hq, D], k8/v8 [B, Sk, Hkv,
 *   D] bytes (or packed [total, H, D] with cu_seqlens as gqa_attn_fwd); D = 128;
 *   out bf16 like q, lse fp32 as gqa_attn_fwd; causal as gqa_attn_fwd.
 * S = Q K^T and O += P V run as 8-bit tensor-core products (kind::f8f6f4, fp32
 * accumulation); P is rounded to e4m3 (relative to the running row max, times 2^7),
 * O is normalised by the sum of the unrounded p.  Codes 0x7f / 0xff (NaN) are not
 * supported.  Errors as gqa_attn_fwd, plus GQA_ERR_SCALE for a scale that is not
 * finite and positive.
 */
int gqa_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, void* out, float* lse,
                     int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, float q_scale,
                     float k_scale, float v_scale, int causal, const int* cu_seqlens,
                     cudaStream_t stream);

/*
 * Block-sparse attention over packed variable-length sequences with minimum padding
 * (Raptor-T abstract: BigBird's block-sparse attention; the minimum-padding algorithm
 * pads each sequence only to whole blocks instead of to the longest sequence; the
 * attention-balancing algorithm assigns thread-block work by its execution time).
 *   q, out [total, Hq, D], k, v [total, Hkv, D] bf16 packed as gqa_attn_fwd's varlen
 *   form; lse [Hq, total]; cu_seqlens device int32 [B + 1]; self attention within each
 *   sequence, causal (key j visible to query i only if j <= i) when causal != 0;
 *   sequence b owns ceil(n_b / 128) query and key blocks (the last one partial);
 *   blk_off device int32 [B + 1]: its first pattern row, the prefix sum of those counts;
 *   blk_row_ptr device int32 [blk_off[B] + 1], blk_col device int32: the CSR pattern,
 *   rows in sequence order, col entries counting the sequence's own key blocks (an
 *   entry outside them raises device error 2 and block 0 is read in its place);
 *   tile_order (optional, device int32 [n_order], n_order a multiple of order_grid):
 *   the tile each step of the persistent grid of order_grid CTAs takes, as written by
 *   gqa_attn_sparse_varlen_schedule; nullptr: the varlen longest-first order.
 * PackGQA always; G = Hq / Hkv >= 2 dividing 128 (GQA_ERR_UNSUPPORTED otherwise); D 64
 * or 128; errors as gqa_attn_fwd.
 */
int gqa_attn_fwd_blocksparse_varlen(const void* q, const void* k, const void* v, void* out,
                                    float* lse, const int* cu_seqlens, const int* blk_off,
                                    int B, int Hq, int Hkv, int max_seqlen, int total, int D,
                                    float scale, int causal, const int* blk_row_ptr,
                                    const int* blk_col, const int* tile_order, int n_order,
                                    int order_grid, cudaStream_t stream);

/*
 * Host-side schedule for gqa_attn_fwd_blocksparse_varlen (no device work).  From host
 * copies of cu_seqlens [B + 1] and blk_row_ptr, writes blk_off [B + 1] (host) and the
 * tile order: every (sequence, KV head, position tile) with a cost of its row's key
 * blocks times its occupied sub-tiles plus one, assigned longest first to the least
 * loaded of `grid` CTAs (grid is capped at the number of tiles); CTA c's k-th tile goes
 * to order[k * g + c], unused slots -1.  *order_grid receives g (grid capped at the
 * number of tiles: the launch's order_grid) and *n_order the entries needed (g times
 * the longest list); GQA_ERR_WORKSPACE if order_cap is smaller (call with
 * order_cap = 0 to size it).
 */
int gqa_attn_sparse_varlen_schedule(const int* cu_seqlens, const int* blk_row_ptr, int B,
                                    int Hq, int Hkv, int max_seqlen, int grid, int* blk_off,
                                    int* order, int order_cap, int* n_order, int* order_grid);

/*
 * Decode (one new query position per sequence) against a KV cache, with per-
 * sequence cache lengths and an optional sliding window.  Ultralytics glossary
 * "Grouped Query Attention (GQA)": during generation the model keeps the keys and
 * values of every earlier token in the KV cache and reads all of it for each new
 * token ("How GQA shrinks the KV cache"); sliding-window attention caps the tokens
 * each layer attends to ("GQA and related techniques").
 *
 * For sequence b with L = seqlens_k[b] cached keys (seqlens_k NULL: L = Sk for
 * every sequence) and query head h, with c = h / (Hq / Hkv):
 *   keys j in [j0, L), j0 = max(0, L - window) if window > 0, else 0;
 *   out[b, h, :] = sum_j softmax_j(scale * q[b,h,:] . k[b,j,c,:]) v[b,j,c,:]
 *   lse[b, h]    = ln sum_j exp(scale * q[b,h,:] . k[b,j,c,:])
 * A sequence with no key (L = 0) gets out = 0 and lse = -inf.
 *
 * Layouts (device pointers, caller-owned, bf16 unless noted):
 *   q, out [B, 1, Hq, D]; lse [B, Hq, 1] fp32;
 *   k_cache, v_cache [B, Sk, Hkv, D]: Sk keys of capacity per sequence, the first
 *     L of them valid;
 *   seqlens_k: NULL or device int32 [B] with 0 <= seqlens_k[b] <= Sk; a value
 *     outside that range raises device error 3 and is clamped.
 * max_seqlen_k (host): an upper bound of seqlens_k (<= Sk), used to choose
 *   num_splits; ignored when seqlens_k is NULL.  window >= 0 (0: every key).
 * num_splits (0 = automatic, from min(max_seqlen_k, window + 64) keys) and
 *   pack_gqa as for gqa_attn_fwd's decode; each sequence divides its own key range
 *   into the splits.  D 64 or 128.  Nothing is allocated or synchronised; with
 *   num_splits > 1 the registered workspace must hold
 *   gqa_attn_workspace_bytes(B, Hq, 1, D, num_splits).
 * Returns gqa_attn_fwd's status codes (GQA_ERR_SHAPE also for window < 0,
 *   max_seqlen_k > Sk).
 */
int gqa_attn_decode_kvcache(const void* q, const void* k_cache, const void* v_cache,
                            const int* seqlens_k, void* out, float* lse, int B, int Hq, int Hkv,
                            int Sk, int D, int max_seqlen_k, float scale, int window,
                            int num_splits, int pack_gqa, cudaStream_t stream);

/*
 * The same decode against a paged KV cache (PagedAttention, Ultralytics glossary
 * "GQA and related techniques": the cache is allocated in fixed-size blocks).
 *   k_pages, v_pages [num_pages, page_size, Hkv, D]: a pool of pages;
 *   block_table: device int32 [B, max_pages]; key j of sequence b is row
 *     j % page_size of page block_table[b * max_pages + j / page_size];
 *   seqlens_k: device int32 [B] (required), 0 <= seqlens_k[b] <= max_pages *
 *     page_size.  Only the table entries of pages holding keys j < seqlens_k[b]
 *     are read; an entry outside [0, num_pages) raises device error 3 and page 0
 *     is read in its place.
 *   page_size: a power of two >= 16; num_pages * page_size < 2^31.
 * Everything else (window, max_seqlen_k <= max_pages * page_size, num_splits,
 * pack_gqa, q/out/lse layouts, workspace, errors) as gqa_attn_decode_kvcache.
 */
int gqa_attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                          const int* block_table, const int* seqlens_k, void* out, float* lse,
                          int B, int Hq, int Hkv, int D, int num_pages, int page_size,
                          int max_pages, int max_seqlen_k, float scale, int window,
                          int num_splits, int pack_gqa, cudaStream_t stream);

/*
 * The same decode against a KV cache stored in 8 bits: every K and V element is an
 * e4m3 code (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; subnormals below
 * 2^-6; largest finite 448; the NaN codes 0x7f and 0xff are not propagated: they are
 * read as +-480), and the stored value is
 * code_value * k_scale (keys) or code_value * v_scale (values), one scale per tensor.
 * The attention is gqa_attn_decode_kvcache's on those decoded values.  The GQA
 * batch-size guide names FP8 as the way to lower memory-bandwidth pressure (hardware
 * adaptation section, Hopper item; precision row of its production checklist); the
 * cache is read once in 8 bits, half the bytes of bf16.
 *   block_table NULL: k8, v8 [B, Sk, Hkv, D] uint8 codes (num_pages, page_size and
 *     max_pages ignored);
 *   block_table given: k8, v8 [num_pages, page_size, Hkv, D] codes with
 *     gqa_attn_decode_paged's table, lengths and page rules (Sk ignored);
 *   q bf16 [B, 1, Hq, D] (rounded to f16 for the products: |q| must stay below
 *     65504), out bf16 [B, 1, Hq, D], lse fp32 [B, Hq, 1]; k_scale, v_scale finite
 *     and > 0 (GQA_ERR_SCALE otherwise).
 * num_splits = 0 chooses up to 64 splits for two resident CTAs per SM (the 8-bit path
 * converts every element and needs the extra warps): the count with the shortest
 * estimated makespan, whole waves of equal splits each costing its 64-key blocks plus
 * about three; a registered workspace of gqa_attn_workspace_bytes(B, Hq, 1, D, 64)
 * always suffices.  Status codes, window,
 * explicit splits and pack_gqa as gqa_attn_decode_kvcache.
 */
int gqa_attn_decode_fp8(const void* q, const void* k8, const void* v8, float k_scale,
                        float v_scale, const int* block_table, const int* seqlens_k, void* out,
                        float* lse, int B, int Hq, int Hkv, int D, int Sk, int num_pages,
                        int page_size, int max_pages, int max_seqlen_k, float scale, int window,
                        int num_splits, int pack_gqa, cudaStream_t stream);

/*
 * Diagnostic: exercises the kernels' bounded-wait path.  Launches one warp that
 * waits, with the same bounded mbarrier wait the attention kernels use, on a
 * barrier nothing completes; after limit_ms (1..1000) the wait gives up, records
 * device error 1 (wait timed out) and the kernel returns, leaving the context
 * usable.  Read the code with gqa_attn_get_device_error.  Nothing faults or traps.
 */
int gqa_attn_selftest_timeout(int limit_ms, cudaStream_t stream);

/* Static description of a status code. */
const char* gqa_attn_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* GQA_ATTN_H */
