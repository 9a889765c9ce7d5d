/*
 * ssta.h — C ABI of the SSTA forward library (libssta.so) for NVIDIA B200 (sm_100a).
 *
 * Selective and Sliding Tile Attention (SSTA) is the block-sparse self-attention
 * over the 3D (latent frame x height x width) token grid of a video diffusion
 * transformer, described in "HunyuanVideo 1.5 Technical Report" (paper-graph-ui
 * summary), section "SSTA: Selective and Sliding Tile Attention", in four steps:
 *   Step 1  3D Block Partition                     -> ssta_tile_reorder
 *   Step 2  Selective Mask Generation (top-k)      -> ssta_build_block_mask
 *   Step 3  STA sliding tile window mask           -> ssta_build_block_mask
 *   Step 4  Combine masks + block-sparse attention -> ssta_build_block_mask (union,
 *                                                     compact lists) and
 *                                                     ssta_attention_fwd
 * plus ssta_tile_unorder, the inverse layout change of Step 1.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Memory: every tensor argument is a DEVICE pointer to caller-owned, dense,
 *    row-major storage.  The library never allocates, frees or synchronises;
 *    each call only enqueues kernels on `stream` (a cudaStream_t passed as
 *    void*, NULL = the legacy default stream) and returns.
 *  - Alignment: tensor pointers must be 16-byte aligned, the workspace 256-byte
 *    aligned; otherwise SSTA_ERR_ALIGNMENT.
 *  - Errors: arguments are checked on the host before anything is launched.
 *    Launch failures return SSTA_ERR_LAUNCH.  Faults the kernels detect on the
 *    device (an out-of-range kept-tile id, a pipeline wait that exceeded its
 *    time limit, or - in the backward dK/dV kernel, whose shared-memory layout
 *    leaves under 1 KB to align its base - a dynamic shared-memory base the
 *    runtime did not place 1024-byte aligned, SSTA_ERR_ALIGNMENT) do not trap:
 *    the kernel records a code in the first 4 bytes of the workspace (an int32;
 *    0 = no error, else an ssta_status value) and returns; read it with
 *    ssta_read_device_status after the stream completes.
 *  - Calls are stateless and thread-safe; separate calls may run concurrently
 *    on different streams if their workspaces differ.
 *  - Dtypes: SSTA_BF16 (bfloat16 storage; tensor-core attention with fp32
 *    softmax and accumulation) or SSTA_F32 (fp32 storage and arithmetic).
 *
 * Layouts (B = batch, H = heads, D = head dim = 128)
 * --------------------------------------------------
 *  raster  [B, H, T, Y, X, D]     tokens of the valid latent grid.
 *  text    [B, H, L_text, D]      optional text tokens (L_text may be 0).
 *  packed  [B, H, Lq, D]          Lq = NT*N + L_text.  The grid is padded up to
 *          whole tiles (tT x tY x tX tokens, N = tT*tY*tX); video tile
 *          c = (cT*nY + cY)*nX + cX owns rows c*N .. c*N+N-1 with its tokens in
 *          raster order; pad rows are zero; text rows follow all video tiles.
 *  kv_idx  [B, H, NQ, max_kept] int32, NQ = NT + ceil(L_text/N) query tiles; row
 *          (b,h,i) lists the key tiles query tile i attends, ascending, padded
 *          with -1.  Key tiles NT.. are the text tiles.
 *  kv_cnt  [B, H, NQ] int32 number of valid entries of each kv_idx row.
 *  lse     [B, H, Lq] fp32, natural-log sum of exp of the scaled scores of a row.
 */
#ifndef SSTA_H
#define SSTA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSTA_OK = 0,
  SSTA_ERR_INVALID_ARG = 1,    /* NULL pointer, negative or zero size, bad field */
  SSTA_ERR_UNSUPPORTED = 2,    /* well-formed but outside what the kernels implement */
  SSTA_ERR_ALIGNMENT = 3,      /* pointer not 16-byte (tensors) / 256-byte (workspace) aligned */
  SSTA_ERR_WORKSPACE = 4,      /* workspace NULL or smaller than ssta_plan's workspace_bytes */
  SSTA_ERR_LAUNCH = 5,         /* CUDA refused a launch (see cudaGetLastError) */
  SSTA_ERR_DEVICE_TIMEOUT = 6, /* device code: a pipeline wait exceeded its limit */
  SSTA_ERR_DEVICE_BOUNDS = 7   /* device code: a kept-tile id or count was out of range */
} ssta_status;

typedef enum { SSTA_BF16 = 0, SSTA_F32 = 1 } ssta_dtype;

/* Block score ranked by top-k (Step 2, "Selective Mask Generation"). */
typedef enum {
  SSTA_SCORE_SIMILARITY = 0, /* Score_s = Qbar . Kbar (raw dot product of the tile means) */
  SSTA_SCORE_IMPORTANCE = 1  /* lambda (cos(Qbar, Kbar) + 1) / 2 - (1 - lambda) * redundancy, where the
                                redundancy of key tile j is the mean over the other key tiles j' of
                                (cos(Kbar_j', Kbar_j) + 1) / 2 (0 when NT = 1); an all-zero mean has
                                cosine 0 with everything */
} ssta_score_mode;

/* How selection and window combine (Step 4). */
typedef enum {
  SSTA_COMBINE_UNION = 0,    /* selected OR in the window */
  SSTA_COMBINE_AND = 1       /* selected AND in the window (Algorithm 1 as printed) */
} ssta_combine;

/* Window at the grid edges (Step 3).  The window of tile c on an axis of n tiles
 * covers [c - w/2, c - w/2 + w) (integer w/2). */
typedef enum {
  SSTA_WINDOW_SHIFT = 0,     /* slid inward so it keeps min(w, n) tiles */
  SSTA_WINDOW_TRUNCATE = 1   /* cut at 0 and n */
} ssta_window;

/* Problem descriptor.  All fields are plain integers or floats; see the layouts
 * above.  A descriptor whose mode fields are all zero selects the similarity
 * score, the union and the shifted window. */
typedef struct {
  int B, H, D;      /* batch, heads, head dim (D must be 128) */
  int T, Y, X;      /* valid latent grid: frames, height, width (each >= 1) */
  int tT, tY, tX;   /* tile extent per axis in tokens (each >= 1) */
  int wT, wY, wX;   /* sliding window per axis, in tiles (each >= 1; odd = centred) */
  int topk;         /* key tiles selected per query tile (>= 0; clamped to NT) */
  int L_text;       /* appended text tokens (>= 0) */
  int dtype;        /* ssta_dtype */
  float scale;      /* softmax scale; 0 means 1/sqrt(D) */
  int score_mode;   /* ssta_score_mode */
  float lambda;     /* importance score: weight of the similarity term, in [0, 1] (the pages use 0.9);
                       ignored by the similarity score */
  int combine;      /* ssta_combine */
  int window_mode;  /* ssta_window */
} ssta_desc;

/* Sizes derived from a descriptor. */
typedef struct {
  int64_t packed_len;      /* Lq */
  int num_tiles;           /* NT video tiles */
  int num_text_tiles;      /* ceil(L_text / N) */
  int num_q_tiles;         /* NQ = NT + num_text_tiles */
  int tile_tokens;         /* N */
  int topk;                /* min(topk, NT) */
  int window_tiles;        /* prod over axes of min(w, n) */
  int max_kept;            /* row width of kv_idx */
  size_t workspace_bytes;  /* workspace for ssta_build_block_mask (>= 256) */
  size_t attn_workspace_bytes; /* workspace for ssta_attention_fwd (256) */
  size_t bwd_workspace_bytes;  /* workspace for ssta_attention_bwd */
} ssta_plan_info;

/*
 * ssta_plan — derive every size from `desc` (host only, no CUDA call).
 * Step 1, "3D Block Partition": NT = ceil(T/tT)*ceil(Y/tY)*ceil(X/tX).
 * max_kept = NT + num_text_tiles when L_text > 0 (text query tiles attend every
 * tile), else min(NT, topk + window_tiles).  window_tiles is the largest window
 * (with SSTA_WINDOW_TRUNCATE edge tiles keep fewer).  workspace_bytes depends on
 * score_mode (the importance score keeps per-tile norms and redundancies).
 * Returns SSTA_ERR_INVALID_ARG also for an unknown mode or lambda outside [0, 1].
 * Returns SSTA_ERR_INVALID_ARG for malformed descriptors, SSTA_ERR_UNSUPPORTED
 * when D != 128, N > 4096, NT > 2048, B*H > 65535 or Lq >= 2^31.
 */
ssta_status ssta_plan(const ssta_desc* desc, ssta_plan_info* info);

/*
 * ssta_tile_reorder — Step 1 ("3D Block Partition"): gather raster tokens into
 * the packed tile-major layout, zero the pad rows and append the text tokens.
 *   x_raster [B,H,T,Y,X,D] (read), x_text [B,H,L_text,D] (read; NULL iff
 *   L_text == 0), x_packed [B,H,Lq,D] (written in full).  Element type = dtype.
 * Exact copy.  The three buffers must not overlap.
 */
ssta_status ssta_tile_reorder(const ssta_desc* desc, const void* x_raster, const void* x_text,
                              void* x_packed, void* stream);

/*
 * ssta_build_block_mask — Steps 2-4 up to the mask: per (b, h, video tile) mean
 * of q and k over the tile's valid tokens; fp32 block scores (Step 2: Score_s =
 * Qbar Kbar^T, computed on the tensor cores with each fp32 mean split into three
 * bf16 parts and six products accumulated in fp32, or the importance score of
 * desc->score_mode, computed with fp32 FMA); per query tile the
 * top-k key tiles by score, ties to the lower tile index (Step 2,
 * Topk/Indexes2mask); combined (desc->combine: union, or AND) with the sliding
 * tile window (Step 3; desc->window_mode: slid inward at the grid edges so it
 * always spans min(w, n) tiles per axis, or truncated), and with every text tile;
 * text query tiles keep every tile (Step 4).  Writes the compact lists; a video
 * query tile can keep no tile at all (AND, no text), its count is then 0.
 *   q_packed, k_packed [B,H,Lq,D] (read; pad rows are ignored),
 *   kv_idx [B,H,NQ,max_kept] and kv_cnt [B,H,NQ] (written),
 *   tile_scores [B,H,NT,NT] fp32: the block scores top-k ranks (written when
 *   non-NULL, else kept in workspace),
 *   workspace >= info.workspace_bytes (contents overwritten).
 */
ssta_status ssta_build_block_mask(const ssta_desc* desc, const void* q_packed, const void* k_packed,
                                  int32_t* kv_idx, int32_t* kv_cnt, float* tile_scores,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * ssta_attention_fwd — Step 4 ("flex_block_attention"): for every packed query
 * row, softmax(q k^T * scale) v over the valid keys of the kept key tiles of
 * its query tile (full attention inside each kept tile; key tiles that are not
 * listed are never read).  Pad query rows are computed but carry no meaning.
 * A query tile with no valid kept key gets O = 0 and LSE = -inf.
 *   q/k/v_packed [B,H,Lq,D] (read), kv_idx/kv_cnt as written by
 *   ssta_build_block_mask (read; ids must be < NQ and ascending order is not
 *   required), o_packed [B,H,Lq,D] (written, dtype), lse [B,H,Lq] fp32
 *   (written), workspace >= info.attn_workspace_bytes (device status word).
 * bf16: tcgen05 tensor-core kernel; needs N % 128 == 0, else
 * SSTA_ERR_UNSUPPORTED (the paper's 4x8x8 tiles hold 256 tokens).
 * f32: SIMT kernel, any N.
 */
ssta_status ssta_attention_fwd(const ssta_desc* desc, const void* q_packed, const void* k_packed,
                               const void* v_packed, const int32_t* kv_idx, const int32_t* kv_cnt,
                               void* o_packed, float* lse, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * ssta_attention_bwd — gradients of ssta_attention_fwd (Step 4) for training: with
 * P = exp(q k^T * scale - LSE) over the valid keys of each query tile's kept tiles,
 * D = rowsum(dO * O) and dS = P * (dO v^T - D):
 *   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO.
 * Pad query rows take no part (dQ = 0 there); pad key rows get dK = dV = 0.
 *   q/k/v/o/do_packed [B,H,Lq,D] (read; o and lse as ssta_attention_fwd wrote them,
 *   do = dL/dO), kv_idx/kv_cnt as ssta_build_block_mask wrote them (ascending lists
 *   required), dq/dk/dv_packed [B,H,Lq,D] (written in full), all of `dtype`;
 *   workspace >= info.bwd_workspace_bytes (status word, per-row D, per-row -LSE and -D
 *   over whole tiles for the bf16 kernels, and for every key tile the list of query
 *   tiles keeping it).
 * bf16 (N % 128 == 0 required, as for ssta_attention_fwd): tcgen05 tensor-core
 * kernels, one for dQ over each query tile's kept list, one for dK and dV over the
 * query tiles keeping each key tile.  fp32: SIMT kernels with fp32 arithmetic.
 * Returns SSTA_ERR_UNSUPPORTED for bf16 with N % 128 != 0, SSTA_ERR_WORKSPACE for a
 * missing or short workspace, SSTA_ERR_ALIGNMENT for a workspace not 256-byte aligned
 * or a tensor not 16-byte aligned, SSTA_ERR_INVALID_ARG for a NULL tensor.
 */
ssta_status ssta_attention_bwd(const ssta_desc* desc, const void* q_packed, const void* k_packed,
                               const void* v_packed, const void* o_packed, const float* lse,
                               const void* do_packed, const int32_t* kv_idx, const int32_t* kv_cnt,
                               void* dq_packed, void* dk_packed, void* dv_packed, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * ssta_tile_unorder — inverse of ssta_tile_reorder: scatter packed rows back to
 * the raster layout, dropping pad rows, and split off the text rows.
 *   x_packed [B,H,Lq,D] (read), x_raster [B,H,T,Y,X,D] (written),
 *   x_text [B,H,L_text,D] (written; may be NULL to drop the text rows).
 */
ssta_status ssta_tile_unorder(const ssta_desc* desc, const void* x_packed, void* x_raster,
                              void* x_text, void* stream);

/*
 * ssta_build_block_mask_noalloc — the same computation and outputs as
 * ssta_build_block_mask, for callers that cannot allocate device memory at call
 * time (for instance a plugin that an inference engine hands only pre-planned
 * tensors, or a service that reserved all device memory for its own pool).  The
 * paper has no counterpart to this call; it exists for those callers only.
 *   Scratch: a device array of SSTA_STATIC_SCRATCH_BYTES built into the library,
 *   one per GPU that loads it, resident until the process exits.  It holds the
 *   workspace layout of ssta_build_block_mask: a 256-byte header, the pooled q and
 *   k means, in importance mode the inverse norms and the key sums, and the score
 *   matrix unless tile_scores is given.  Problems whose layout exceeds the array
 *   return SSTA_ERR_WORKSPACE.  The mask kernels report no device-side errors and
 *   the array's address is not exported, so this call keeps no device status word
 *   (there is nothing for ssta_read_device_status to read).
 *   The call allocates nothing.  All calls on a device share the array, so calls
 *   whose kernels overlap on the GPU race: serialise them.  The first call on a
 *   device looks up the array's device address (with that device current); make
 *   it before any stream capture.
 *   Arguments as for ssta_build_block_mask, without the workspace.
 */
#define SSTA_STATIC_SCRATCH_BYTES (32u << 20)
ssta_status ssta_build_block_mask_noalloc(const ssta_desc* desc, const void* q_packed, const void* k_packed,
                                          int32_t* kv_idx, int32_t* kv_cnt, float* tile_scores, void* stream);

/*
 * ssta_selftest_bounded_wait — runs the device-side bounded wait that guards every
 * pipeline wait of ssta_attention_fwd on a barrier phase that never completes
 * (complete == 0) or that completes at once (complete != 0).  The paper has no
 * counterpart; this exists to test failure handling without faulting a GPU.
 *   timeout_us in [1, 2,000,000]: the wait's limit; workspace >= 256 bytes.
 * Afterwards the workspace status word (ssta_read_device_status) holds
 * SSTA_ERR_DEVICE_TIMEOUT (never-completing phase, after about timeout_us) or 0.
 */
ssta_status ssta_selftest_bounded_wait(int32_t timeout_us, int32_t complete, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * ssta_read_device_status — copy the device status word (first int32 of a
 * workspace used by the calls above) to *code, synchronising `stream` first.
 * Diagnostic call: the only function of this library that synchronises.
 */
ssta_status ssta_read_device_status(const void* workspace, void* stream, int32_t* code);

/* Static, human-readable name of a status code. */
const char* ssta_status_string(ssta_status status);

#ifdef __cplusplus
}
#endif

#endif /* SSTA_H */
