/*
 * unstep.h -- C ABI of the B200 (sm_100a) chunk-causal attention layer of UnStep's causal video
 * DiT step.
 *
 * Source: "UnStep: Training-Free Acceleration of Causal Video Diffusion with Fewer Steps Than
 * Distillation" (arXiv 2609.32518).  The abstract names the runtime stack of the DiT: RoPE from
 * cached coefficients, KV-cache indexing, more efficient attention calls, and a limit on the
 * temporal window that the attention KV cache retains (Table 1, rows C1 and C4).  Table 3 fixes
 * the stream: seven causal chunks of three latent frames per 81-frame clip.
 *
 * One layer of that step is three operations, exposed as two calls:
 *   unstep_rope_kv_append  -- 3D RoPE of a chunk's q and k from the cached cos/sin tables,
 *                             q rotated in place, rotated k and v written into a ring-buffer KV
 *                             cache that keeps the last cap_frames latent frames (frame f in
 *                             slot f mod cap_frames);
 *   unstep_window_attn     -- softmax attention of that chunk's queries over the last `window`
 *                             latent frames ending at the chunk's last frame (the chunk itself
 *                             included), scale 1/sqrt(D), fp32 accumulation and softmax.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers into memory the caller allocated and owns.  The
 *     library never allocates or frees device memory and keeps no pointer beyond a call, except
 *     the ones the caller stores in unstep_cache_t.
 *   - Work is enqueued on the caller's stream; no call synchronises the stream, except
 *     unstep_cache_init (pageable host->device copy of the tables) and unstep_get_device_error.
 *   - Every call returns UNSTEP_OK (0) or a negative UNSTEP_ERR_* code and never throws.  A call
 *     that fails on the host leaves the cache and every buffer unchanged.
 *   - Tensors are bf16, row-major, densely packed.  Activation layout is [B][L][H][D] (stream,
 *     token, head, channel); token l of a chunk is (i, y, x) with l = i*Hg*Wg + y*Wg + x, i the
 *     frame inside the chunk.  Cache layout is [B][H][cap_frames*Hg*Wg][D]; frame f's token tok
 *     lives in row (f mod cap_frames)*Hg*Wg + tok.
 *   - Pointers must be 16-byte aligned (UNSTEP_ERR_ALIGN otherwise); D must be 64 or 128
 *     (UNSTEP_ERR_UNSUPPORTED).
 *   - An unstep_cache_t may not be used from two host threads at once.
 */
#ifndef UNSTEP_H_
#define UNSTEP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st *unstep_stream_t;

enum {
  UNSTEP_OK = 0,
  UNSTEP_ERR_ARG = -1,            /* NULL pointer, uninitialised cache, bad scalar */
  UNSTEP_ERR_SHAPE = -2,          /* shapes disagree with the cache */
  UNSTEP_ERR_ALIGN = -3,          /* a pointer is not 16-byte aligned */
  UNSTEP_ERR_FRAME_ORDER = -4,    /* frame_idx is neither the next chunk nor the latest chunk */
  UNSTEP_ERR_WINDOW = -5,         /* window outside [chunk frames, cap_frames], or empty cache */
  UNSTEP_ERR_UNSUPPORTED = -6,    /* D not 64/128, or a size beyond the kernels' index range */
  UNSTEP_ERR_CUDA = -7,           /* a CUDA runtime call failed (launch, copy, memset) */
  UNSTEP_ERR_DEVICE_TIMEOUT = -8, /* a kernel gave up waiting (reported by the device word) */
  UNSTEP_ERR_SCRATCH_LIMIT = -9,  /* unstep_window_attn_noalloc: call too large for its buffer */
  UNSTEP_ERR_DEVICE_BOUNDS = -10  /* debug build only: a kernel's index check failed (device word) */
};

/*
 * One layer's KV cache and RoPE coefficient cache.
 * The caller fills the shape fields and the five device pointers, then calls unstep_cache_init,
 * which fills the coefficient tables and the metadata fields.
 */
typedef struct {
  /* shape (caller) */
  int B;            /* independent streams */
  int H;            /* heads */
  int D;            /* head width: 64 or 128 */
  int Hg, Wg;       /* token grid of one latent frame; T_f = Hg*Wg tokens */
  int d_t, d_h, d_w;/* RoPE channel blocks, in this order; each even, sum == D */
  double theta;     /* RoPE base, e.g. 10000 */
  int cap_frames;   /* ring capacity in latent frames (the retained window W) */
  int max_pos_t;    /* temporal positions 0 .. max_pos_t-1 are valid frame indices */
  /* device memory (caller-allocated, caller-owned) */
  void *k_cache;    /* bf16 [B][H][cap_frames*T_f][D] */
  void *v_cache;    /* bf16 [B][H][cap_frames*T_f][D] */
  int *slot_frame;  /* int32 [cap_frames]: frame held by each slot, -1 = empty */
  float *cos_sin;   /* fp32 coefficient tables, unstep_cache_table_bytes() bytes */
  int *dev_error;   /* int32 [1]: first device-side error, 0 = none */
  /* optional attention scratch (caller-allocated, caller-owned; may be NULL): with it,
   * unstep_window_attn balances its work over all SMs by splitting some (head, query) units
   * along keys; without it, one CTA per unit.  unstep_attn_scratch_bytes() bytes, 16-byte
   * aligned.  Several caches may share one scratch buffer if their attention calls never
   * overlap on the GPU (e.g. they are issued on one stream). */
  void *attn_scratch;
  size_t attn_scratch_bytes;
  /* metadata (library-maintained; read-only for the caller) */
  int frames_written;    /* one past the newest frame written */
  int first_frame;       /* temporal position of the stream's first frame */
  int last_chunk_start;  /* first frame of the latest chunk, -1 before any */
  int last_chunk_frames; /* frames of the latest chunk, 0 before any */
  int initialized;       /* set by unstep_cache_init */
  /* shard of the activations (caller; all zero = the cache covers the whole activation tensor).
   * Streams and heads are independent in every step of the layer (the paper's window is per
   * stream and head), so a layer splits over GPUs by (stream, head) ranges with no exchange.
   * This cache then holds streams b0 .. b0+B-1 and heads h0 .. h0+H-1 of activations laid out
   * as [act_B][L][act_H][D]: q, k, v and out are those full tensors, and every call reads and
   * writes only this shard's rows of them, in place.  act_B = 0 means B, act_H = 0 means H;
   * 0 <= b0, b0 + B <= act_B, 0 <= h0, h0 + H <= act_H, act_B * act_H <= 2^30. */
  int act_B, act_H;
  int b0, h0;
} unstep_cache_t;

/* The chunk a call covers: `frames` latent frames of Hg x Wg tokens. */
typedef struct {
  int frames, Hg, Wg;
} unstep_grid_t;

/* Resolved key set of a window: at most two contiguous row ranges of the ring. */
typedef struct {
  int first_frame, last_frame; /* frames attended, inclusive */
  int keys;                    /* (last_frame - first_frame + 1) * T_f */
  int seg_row[2];              /* first cache row of each range */
  int seg_len[2];              /* rows in each range; seg_len[1] == 0 when the range is one */
} unstep_window_plan_t;

/* Library version, e.g. 101 for 0.1.1. */
int unstep_version(void);

/* Text for a status code (static storage). */
const char *unstep_status_string(int status);

/* Bytes the caller must allocate for cache->cos_sin (0 if the shape fields are invalid).
 * Layout: float2 (cos, sin) tables, temporal [max_pos_t][d_t/2], then height [Hg][d_h/2], then
 * width [Wg][d_w/2]; entry j of position pos holds cos/sin of pos * theta^(-2j/d_a). */
size_t unstep_cache_table_bytes(const unstep_cache_t *cache);

/* Bytes of ONE of k_cache / v_cache for this shape (0 if invalid). */
size_t unstep_cache_kv_bytes(const unstep_cache_t *cache);

/* Bytes of the optional attention scratch for this shape on the CURRENT device (it depends on
 * the device's SM count): per-(unit, query tile) counters plus two slots per SM of
 * 2 x (D x 128 + 256) floats.  0 if the shape fields are invalid or no device is usable. */
size_t unstep_attn_scratch_bytes(const unstep_cache_t *cache);

/*
 * Validate the shape fields and pointers, compute the coefficient tables on the host in fp64,
 * round them to fp32 and copy them to cache->cos_sin; zero k_cache, v_cache, dev_error and the
 * scratch counters; set every slot_frame entry to -1; reset the metadata.  Enqueued on `stream`;
 * the table copy is from pageable memory, so the call returns only after the copy has been
 * staged.
 * Errors: ARG (NULL pointers, odd or negative split, split sum != D, cap_frames < 1,
 * max_pos_t < 1, theta <= 0, attn_scratch_bytes too small), UNSUPPORTED (D not 64/128, sizes
 * beyond 32-bit row indexing), ALIGN, CUDA.
 */
int unstep_cache_init(unstep_cache_t *cache, unstep_stream_t stream);

/*
 * Host-only check of an append: the slots frames frame_idx .. frame_idx+grid.frames-1 would
 * occupy (written to slots_out[0 .. grid.frames-1] if slots_out is non-NULL), and whether the
 * append is a new chunk (returns 1) or a re-forward of the latest chunk (returns 0).
 * Rules: grid.Hg/Wg equal the cache's, 1 <= grid.frames <= cap_frames, the frames lie in
 * [0, max_pos_t); frame_idx is either frames_written (next chunk; any frame_idx >= 0 for the
 * stream's first chunk) or last_chunk_start with the same frame count (a later denoising step or
 * the clean-cache pass of the same chunk, which overwrites the same slots).
 * Errors: ARG, SHAPE, FRAME_ORDER, WINDOW (grid.frames > cap_frames).  Touches no GPU state.
 */
int unstep_append_plan(const unstep_cache_t *cache, int frame_idx, unstep_grid_t grid,
                       int *slots_out);

/*
 * Fused 3D RoPE + KV-cache append of one chunk (all B streams at the same frame_idx).
 *   q  : bf16 [B][L][H][D], L = grid.frames*Hg*Wg; rotated IN PLACE.
 *   k  : bf16 [B][L][H][D], read only; its rotation goes to k_cache.
 *   v  : bf16 [B][L][H][D], read only; copied bit-exactly to v_cache.
 * (For a shard cache, act_B and act_H replace B and H in these layouts and only the shard's
 * streams and heads are read and written.)
 * Channel pair (2p, 2p+1) of block a (t, h or w, in that channel order) with in-block index j is
 * rotated by +ang, ang = pos_a * theta^(-2j/d_a), pos_t = absolute frame index, pos_h = y,
 * pos_w = x, in fp32 from the fp32 tables, results rounded to bf16 (RNE).  Writes
 * slot_frame[f mod cap] = f for the chunk's frames and then updates the metadata.
 * Errors: those of unstep_append_plan, plus ALIGN and CUDA.
 */
int unstep_rope_kv_append(void *q, const void *k, const void *v, unstep_cache_t *cache,
                          int frame_idx, unstep_grid_t grid, unstep_stream_t stream);

/*
 * Flags of unstep_rope_kv_append_ex.
 *   UNSTEP_APPEND_DEFER_Q_ROPE: q is neither read nor written (it may be NULL); only k and v
 *   are processed (4 of the 6 HBM streams).  The chunk's queries are then rotated by
 *   unstep_window_attn_ex with UNSTEP_ATTN_ROPE_Q, inside the attention.
 */
#define UNSTEP_APPEND_DEFER_Q_ROPE 1u

/*
 * unstep_rope_kv_append with flags (0 = exactly unstep_rope_kv_append).
 * Source: the paper's abstract (RoPE from cached coefficients, KV-cache indexing); applying the
 * query half of the RoPE inside the attention call instead of in the append is this library's
 * own fusion, which saves the round trip of q through HBM.  With UNSTEP_APPEND_DEFER_Q_ROPE the
 * cache, slot_frame and metadata are updated exactly as without it, bit for bit, and q is
 * untouched.
 * Errors: those of unstep_rope_kv_append, plus ARG for an unknown flag bit.
 */
int unstep_rope_kv_append_ex(void *q, const void *k, const void *v, unstep_cache_t *cache,
                             int frame_idx, unstep_grid_t grid, unsigned flags,
                             unstep_stream_t stream);

/*
 * Host-only window resolution for the latest chunk: the frames
 * [max(first_frame, f_end - window + 1), f_end], f_end the latest chunk's last frame, as at
 * most two contiguous row ranges of the ring.  Errors: ARG, WINDOW (no chunk appended yet, or
 * window outside [last_chunk_frames, cap_frames]).
 */
int unstep_window_plan(const unstep_cache_t *cache, int window, unstep_window_plan_t *plan);

/*
 * Windowed chunk-causal attention of the latest chunk.
 *   q   : bf16 [B][L][H][D], the chunk's ROTATED queries (as unstep_rope_kv_append left them),
 *         L = last_chunk_frames*Hg*Wg.
 *   out : bf16 [B][L][H][D]; must not overlap q or the caches.
 *   (For a shard cache, act_B and act_H replace B and H; only the shard's rows of out are
 *   written.)
 * out = softmax(q K^T / sqrt(D)) V over the window's keys (unstep_window_plan), every query of
 * the chunk seeing the same keys.  bf16 tensor-core products with fp32 accumulation, fp32
 * online softmax, output rounded to bf16 (RNE).
 * Errors: ARG, WINDOW, ALIGN, UNSUPPORTED, CUDA.  A device-side wait that runs past its limit
 * sets *dev_error (read it with unstep_get_device_error).
 */
int unstep_window_attn(const void *q, const unstep_cache_t *cache, int window, void *out,
                       unstep_stream_t stream);

/*
 * Flags of unstep_window_attn_ex.
 *   UNSTEP_ATTN_ROPE_Q: q holds the latest chunk's UN-rotated queries (as produced by the
 *   projection); the kernel rotates each query tile after loading it, with the cache's tables and
 *   the positions of the latest appended chunk (frame last_chunk_start + i, grid y, x), exactly
 *   as unstep_rope_kv_append would have rotated it.  q itself is not modified.
 */
#define UNSTEP_ATTN_ROPE_Q 1u

/*
 * unstep_window_attn with flags (0 = exactly unstep_window_attn).
 * With UNSTEP_ATTN_ROPE_Q, the output is bit-identical to unstep_rope_kv_append (q rotated in
 * place) followed by unstep_window_attn on that rotated q, for the same inputs.  Use it after
 * unstep_rope_kv_append_ex with UNSTEP_APPEND_DEFER_Q_ROPE (or after a plain append whose q
 * buffer was a copy).  The query rotation is done by two otherwise idle warps of each CTA.
 * Errors: those of unstep_window_attn, plus ARG for an unknown flag bit.
 */
int unstep_window_attn_ex(const void *q, const unstep_cache_t *cache, int window, void *out,
                          unsigned flags, unstep_stream_t stream);

/*
 * unstep_window_attn for callers that cannot allocate device memory.
 * No counterpart in the paper.  Some callers have no way to call cudaMalloc (code running under
 * a framework or allocator that owns every device allocation, or a process whose device
 * footprint must not grow after start-up), so they cannot provide cache->attn_scratch.  This
 * call computes exactly what unstep_window_attn computes, with the same load-balanced schedule,
 * but keeps its scratch in a buffer that is part of the library itself: 48 MiB of device memory
 * (a file-scope __device__ array) that every GPU which loads the library holds until the process
 * exits.  cache->attn_scratch is ignored.  The call allocates nothing and calls no allocating
 * routine.
 *   - The first call on a device looks up the buffer's device address (with that device current)
 *     and caches it; make that first call before any stream capture.
 *   - Every call on a device uses the same buffer and zeroes the part that must start at zero
 *     (its counters) on `stream` before the kernel.  Calls whose work overlaps on the GPU (two
 *     streams, two threads) race on the buffer: issue them in one stream order.
 *   - Limit: the buffer must hold 2 x (SM count) slots of 2 x (D x 128 + 256) floats plus
 *     8 bytes per (head, 256-query) unit; on a 148-SM B200 with D = 128 that is 37.6 MiB plus the
 *     counters, which covers up to about 1.3 million units.  A larger call returns
 *     UNSTEP_ERR_SCRATCH_LIMIT without doing anything.
 * Errors: those of unstep_window_attn, plus SCRATCH_LIMIT.
 */
int unstep_window_attn_noalloc(const void *q, const unstep_cache_t *cache, int window,
                               void *out, unstep_stream_t stream);

/*
 * Dense GEMM on the tensor cores: C[M][N] = A[M][K] * B[N][K]^T (both operands K-contiguous,
 * nn.Linear's weight layout for B), bf16 in, fp32 accumulation, bf16 RNE out.  Row strides
 * lda, ldb, ldc in elements.  N, K and the strides must be multiples of 8 (16-byte rows for TMA);
 * M, N, K otherwise arbitrary (ragged tiles are zero-filled and not stored).  A device-side wait
 * that runs out sets *dev_error.  Errors: ARG, SHAPE, ALIGN, CUDA.
 */
int unstep_gemm_bf16(const void *a, int lda, const void *b, int ldb, void *c, int ldc, int M,
                     int N, int K, int *dev_error, unstep_stream_t stream);

/*
 * Truncated-SVD projection (UnStep, abstract and Figure 11 / Table 5: truncated SVD of the
 * attention's value and output projections, rank retention 0.92): a linear layer y = x W^T with
 * W [d_out][d_in] ~ U_r S_r V_r^T evaluated through its rank-`rank` factors,
 *   t = x w1^T   (w1 = (V_r S_r)^T, bf16 [rank][d_in]),   y = t w2^T   (w2 = U_r, bf16 [d_out][rank]),
 * as two unstep_gemm_bf16 calls.  x: [M][d_in]; t: caller scratch [M][rank]; y: [M][d_out].
 * rank, d_in and d_out must be multiples of 8 (pad the factors with zero rows/columns: the
 * product is unchanged).  Errors: those of unstep_gemm_bf16.
 */
int unstep_lowrank_linear(const void *x, const void *w1, const void *w2, void *t, void *y, int M,
                          int d_in, int rank, int d_out, int *dev_error, unstep_stream_t stream);

/*
 * Renoise (UnStep, abstract; Tables 4 and 5: the generated latent is renoised to the near-clean
 * level sigma* = 0.02 before the clean-cache pass; a few-step student moves between its
 * denoising steps the same way): out = (1 - sigma) * x0 + sigma * eps elementwise over n bf16
 * values, in fp32 (one fma), rounded to bf16 (RNE).  out may alias x0 or eps.  0 <= sigma <= 1.
 * Errors: ARG, ALIGN, CUDA.
 */
int unstep_renoise(const void *x0, const void *eps, void *out, long long n, float sigma,
                   unstep_stream_t stream);

/*
 * Causal 3x3x3 convolution of a video VAE decoder, channels-last (abstract and Table 1 row C2:
 * the decoder is sped up through its memory layout, precision and convolution kernels).
 *   x    : bf16 [B][T + 2][H][W][C_in]; each stream's first two frames are its causal history
 *          (the last two input frames of the previous chunk, or zeros at the stream's start).
 *   w    : bf16 [C_out][3][3][3][C_in], taps (dt, dy, dx).
 *   bias : fp32 [C_out], or NULL for none.
 *   y    : bf16 [B][T][H][W][C_out]; must not overlap x.
 *   y[b][t][h][x][o] = bias[o] + sum over dt, dy, dx, c of
 *                      w[o][dt][dy][dx][c] * x[b][t + dt][h + dy - 1][x + dx - 1][c],
 * positions outside the frame reading 0: output frame t sees input frames t .. t + 2.  bf16
 * tensor-core products with fp32 accumulation, output rounded to bf16 (RNE).
 *   scratch, scratch_bytes : optional (caller-allocated, caller-owned; NULL and 0 for none).
 *          With it, the output tiles that do not fill a last whole wave of the SMs are cut
 *          along K over all SMs (stream-K); without it they run whole, one per SM.  At least
 *          unstep_conv3d_scratch_bytes() bytes, 16-byte aligned, ZERO-FILLED by the caller before
 *          its first use; every call leaves it fit for the next one, including a call whose
 *          device wait timed out.  Calls that share one scratch buffer must not run at the same
 *          time (same stream, or ordered by events).  The result does not depend on whether
 *          scratch is given, up to the fp32 summation order of the split tiles.
 * Errors: ARG (NULL pointer, size < 1, scratch_bytes too small), ALIGN (x, w, y, scratch not
 * 16-byte aligned, bias not 4-byte), UNSUPPORTED (C_in not a multiple of 64, C_out not a
 * multiple of 8, sizes beyond the kernel's 32-bit tile indexing), CUDA.  A device-side wait past
 * its limit sets *dev_error.
 */
int unstep_conv3d_causal(const void *x, const void *w, const float *bias, void *y, int B, int T,
                         int H, int W, int C_in, int C_out, void *scratch, size_t scratch_bytes,
                         int *dev_error, unstep_stream_t stream);

/* Bytes of unstep_conv3d_causal's optional scratch on the CURRENT device (it depends on the
 * device's SM count, not on the shape); 0 if the device cannot be queried. */
size_t unstep_conv3d_scratch_bytes(void);

/*
 * Checkpoint and resume of a stream's layer state.
 * A causal video stream is generated chunk by chunk in order (paper, Table 3: seven causal
 * chunks per clip); between two chunks all the state a layer carries forward is its ring of
 * K/V rows, slot_frame and the frame-order metadata.  These calls move exactly that state to
 * and from a host buffer, so that a stream can be paused, moved to another device or process,
 * and continued with results bit-identical to an uninterrupted run.  The coefficient tables
 * are not part of the state: they follow from the shape and are rebuilt by unstep_cache_init.
 *
 * Buffer layout (byte offsets, all in the host's byte order):
 *   0   int32 magic "USTC", int32 layout version (1)
 *   8   int32 B, H, D, Hg, Wg, d_t, d_h, d_w, cap_frames, max_pos_t, act_B, act_H, b0, h0
 *   64  double theta
 *   72  int32 frames_written, first_frame, last_chunk_start, last_chunk_frames
 *   88  (padding to 128)
 *   128 int32 slot_frame[cap_frames], padded to a multiple of 16 bytes
 *   then k_cache, then v_cache (unstep_cache_kv_bytes() each, the device layout verbatim)
 * act_B and act_H are stored as the shard extents in use (B and H when unsharded).
 */

/* Bytes of a state buffer for this cache's shape (0 if the shape fields are invalid). */
size_t unstep_cache_state_bytes(const unstep_cache_t *cache);

/*
 * Enqueue on `stream` the copies of the cache's state into host_dst (bytes >= the state size;
 * pinned memory lets the copies run asynchronously, pageable memory makes them synchronous).
 * The buffer is complete once the stream has reached this point: synchronise before reading it.
 * Errors: ARG (uninitialised cache, NULL buffer, too small), CUDA.
 */
int unstep_cache_save(const unstep_cache_t *cache, void *host_dst, size_t bytes,
                      unstep_stream_t stream);

/*
 * Restore a state written by unstep_cache_save into an initialised cache of the same shape
 * (same B, H, D, Hg, Wg, RoPE split, theta, cap_frames, max_pos_t and shard): the K/V rows and
 * slot_frame are copied to the device on `stream` and the metadata set on the host, so the next
 * append continues the saved stream.  The host buffer must stay unchanged until the stream has
 * passed this point.  A buffer whose header does not match is refused before anything is copied.
 * Errors: ARG (uninitialised cache, NULL or short buffer, bad magic or version), SHAPE (shape
 * mismatch), CUDA.
 */
int unstep_cache_restore(unstep_cache_t *cache, const void *host_src, size_t bytes,
                         unstep_stream_t stream);

/*
 * Synchronises `stream`, reads *cache->dev_error and returns it (UNSTEP_OK if no kernel reported
 * an error); CUDA if the copy or the synchronisation itself failed.
 */
int unstep_get_device_error(const unstep_cache_t *cache, unstep_stream_t stream);

/*
 * Self-test of the bounded device wait: launches one CTA that waits on a shared-memory barrier
 * nothing ever completes, giving up after limit_ns nanoseconds; the kernel then writes
 * UNSTEP_ERR_DEVICE_TIMEOUT to *dev_error (int32 device word) and returns normally, leaving the
 * context usable.  Errors: ARG, CUDA.
 */
int unstep_selftest_wait_timeout(int *dev_error, uint64_t limit_ns, unstep_stream_t stream);

/*
 * Self-test of the attention kernel's two base-2 exponentials on n device floats x (fp32):
 * y_poly[i] = the FMA-pipe polynomial (exact range split x = n + f, degree-3 minimax fit of
 * 2^f on [-1/2, 1/2]; inputs below -125 are clamped to -125), y_mufu[i] = the hardware ex2.approx.
 * No counterpart in the paper: it lets a test bound the polynomial's error against both CUDA's
 * instruction and the exact value.  Errors: ARG, CUDA.
 */
int unstep_selftest_exp2(const float *x, float *y_poly, float *y_mufu, int n,
                         unstep_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* UNSTEP_H_ */
