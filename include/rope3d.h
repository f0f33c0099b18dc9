/*
 * rope3d.h -- C ABI of the fused QK-RMSNorm + causal 3D RoPE + KV-cache append
 * library for NVIDIA B200 (sm_100a), librope3d.so.
 *
 * The operation is the per-chunk Q/K preparation step of a causal autoregressive
 * video DiT under "Causal-RoPE SP", from "Accelerating Video Generation Inference
 * with Sequential-Parallel 3D Positional Encoding Using a Global Time Index"
 * (Yuan & Li):
 *   - every token's (t, h, w) comes from its global sequence index i and the
 *     chunk's start frame s (Section 3.3.2 item 1; Section 3.3.3):
 *       t_g = s + floor(i / (H W)),  h = floor(i / W) mod H,  w = i mod W;
 *   - the rotation is a complex multiply x' = x * e^{i(t_g th_T + h th_H + w th_W)}
 *     on adjacent element pairs (2j, 2j+1) = (re, im) of each head (Section 3.3.1,
 *     Section 3.3.2 item 2, Algorithm 2), pairs 0..n_t-1 turning with t_g, the next
 *     n_h with h and the last n_w with w;
 *   - the rotated K and the raw V are written to the KV cache (Algorithm 1 and 3,
 *     step 5), here at cache row (slot + i) mod cache_tokens of a rolling window.
 * Before the rotation q and k each go through RMSNorm over the token's whole
 * N*D feature vector, y = x / sqrt(mean(x^2) + eps) * weight (QK-RMSNorm of the
 * Wan2.1-style backbone; the paper's pages do not state it).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers on the current CUDA device, contiguous,
 *     16-byte aligned.  The caller owns them and the stream; the library owns only
 *     what rope3d_tables_init allocates.
 *   - Work is enqueued on cuda_stream (a cudaStream_t; NULL = the legacy default
 *     stream) and returns without synchronising.  No allocation happens per call.
 *   - Arguments are checked on the host before anything is enqueued; a negative
 *     status means nothing was launched and no output was touched.  A launch
 *     failure reports ROPE3D_ECUDA.  No exception crosses the ABI, nothing aborts,
 *     no device code traps.  rope3d_last_error() gives the reason in words for the
 *     calling thread's most recent failure.
 *   - Layouts: activations [B][n_tok][N][D] with n_tok = token_end - token_begin,
 *     input row r holding global index token_begin + r; caches [B][cache_tokens][N][D].
 *     D must be 128 = 2 (n_t + n_h + n_w) for the tables it was built with.
 *   - Results do not depend on how [0, T*H*W) is cut into token ranges: a range
 *     processed alone is bit-identical to the same rows of a whole-sequence call.
 */
#ifndef ROPE3D_H
#define ROPE3D_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define ROPE3D_API __attribute__((visibility("default")))
#else
#define ROPE3D_API
#endif

/* Status codes. */
#define ROPE3D_OK 0
#define ROPE3D_EINVAL (-1)   /* a size, count, enum or null pointer is invalid        */
#define ROPE3D_ERANGE (-2)   /* an index range exceeds the grid, cache or tables      */
#define ROPE3D_ECUDA (-3)    /* the CUDA runtime reported an error                    */
#define ROPE3D_EDEVICE (-4)  /* no sm_100 device, or the tables live on another device */
#define ROPE3D_EALIGN (-5)   /* a tensor pointer is not 16-byte aligned                */
#define ROPE3D_EOVERLAP (-6) /* output buffers overlap each other or an input          */
#define ROPE3D_ETIMEOUT (-7) /* a kernel gave up a bounded wait (see check_device_status) */
#define ROPE3D_EINDEX (-8)   /* checked build: a kernel skipped an out-of-extent row */

/* Element types of q, k, v, q_out and the caches (all the same type). */
#define ROPE3D_F32 0
#define ROPE3D_BF16 1

/* Frequency schedules (the paper names per-axis frequencies theta_T, theta_H,
 * theta_W and three frequency tables, Algorithm 2, but prints no formula):
 *   PER_AXIS  -- pair j of an axis with n_a pairs turns at theta^(-2j / (2 n_a))
 *                per unit position (each axis an ordinary RoPE over its own
 *                sub-dimension; the default);
 *   HEAD_WIDE -- one schedule theta^(-2j / D) over the head's pairs j = 0..D/2-1,
 *                cut into n_t, n_h, n_w contiguous pieces. */
#define ROPE3D_SCHEDULE_PER_AXIS 0
#define ROPE3D_SCHEDULE_HEAD_WIDE 1

/* How the kernels obtain cos/sin of each pair's angle. */
#define ROPE3D_TRIG_TABLE 0     /* read the precomputed tables (fp64-built, fp32-stored) */
#define ROPE3D_TRIG_ONTHEFLY 1  /* fp32 angle = position * fp32(inv_freq), then sincosf  */

/* Pairing of a head's 128 elements into 64 complex pairs (Section 3.3.1 sets the two
 * forms side by side):
 *   ADJACENT -- pair j = (x[2j], x[2j+1]) as (re, im): the complex view of Algorithm 2
 *               (Wan2.1); the default;
 *   HALF     -- pair j = (x[j], x[j+64]): the cos/sin "rotate_half" form of Qwen2.5-VL's
 *               M-RoPE (with ROPE3D_SCHEDULE_HEAD_WIDE and a 16/24/24 split it is that
 *               layout).  Pair j keeps its axis and frequency either way. */
#define ROPE3D_PAIRING_ADJACENT 0
#define ROPE3D_PAIRING_HALF 1

/* KV-cache layouts: TOKEN_MAJOR [B][cache_tokens][N][D] (default; one appended token is
 * one contiguous row) or HEAD_MAJOR [B][N][cache_tokens][D] (each head's keys and values
 * contiguous, as attention kernels read them). */
#define ROPE3D_CACHE_TOKEN_MAJOR 0
#define ROPE3D_CACHE_HEAD_MAJOR 1

/* KV-cache element formats:
 *   SAME     -- the caches have the dtype of q, k, v (default);
 *   FP8_E4M3 -- quantize-on-append: each head of an appended K or V row is stored as
 *               128 FP8 E4M3 codes (1 byte each; the OCP E4M3 format, max 448) with one
 *               fp32 power-of-two scale (as in the OCP microscaling formats): the
 *               smallest 2^e, e >= -126, with amax(|x|) / 2^e <= 448 over the head
 *               (2^-126 for an all-zero head); code = E4M3(x / 2^e) -- an exact scaling -- rounded to nearest
 *               even, saturating.  K is
 *               quantized from its fp32 value after RMSNorm and RoPE.  A reader recovers
 *               x ~ value(code) * scale.  Scales are laid out like the cache rows:
 *               [B][cache_tokens][N] (token-major) or [B][N][cache_tokens] (head-major).
 *               (The pages mention NVFP4 KV-cache quantization on Blackwell without a
 *               format; E4M3 with per-head scales is this library's choice.) */
#define ROPE3D_CACHE_SAME 0
#define ROPE3D_CACHE_FP8_E4M3 1
/*   NVFP4    -- quantize-on-append into NVFP4, the Blackwell 4-bit format (the
 *               LongLive-2.0 abstract names NVFP4 for its KV cache): each block of 16
 *               consecutive elements of a head holds 16 E2M1 codes (magnitudes 0, 0.5, 1,
 *               1.5, 2, 3, 4, 6; two codes per byte, element 2j in the low nibble) and one
 *               E4M3 block scale S, under a per-tensor fp32 scale g (options
 *               nvfp4_k_global / nvfp4_v_global; 0 means 1).  In fp32, each operation
 *               rounded to nearest:  k = 1 / (6 g) per tensor, S = E4M3(amax k) over the
 *               block, r = 1 / (value(S) g) (0 if S is zero), code = E2M1(x r) rounded to
 *               nearest even, saturating at 6.  A reader recovers x ~ value(code) value(S) g.  K is
 *               quantized from its fp32 value after RMSNorm and RoPE, V from the input.
 *               Caches hold D/2 = 64 bytes per (token, head): [B][cache_tokens][N][64]
 *               (token-major) or [B][N][cache_tokens][64]; k_scale / v_scale then point to
 *               BYTE arrays of D/16 = 8 E4M3 block scales per (token, head), laid out like
 *               the cache rows ([B][cache_tokens][N][8] or [B][N][cache_tokens][8]),
 *               8-byte aligned.  The register kernel runs it. */
#define ROPE3D_CACHE_NVFP4 2

/* Options of the _ex entry points; a NULL pointer or a zeroed struct gives the defaults
 * (adjacent pairing, token-major cache of the input dtype), i.e. the plain entry points'
 * behaviour. */
typedef struct rope3d_options {
    int pairing;       /* ROPE3D_PAIRING_*                                          */
    int cache_layout;  /* ROPE3D_CACHE_TOKEN_MAJOR / _HEAD_MAJOR (fused step only)   */
    int cache_dtype;   /* ROPE3D_CACHE_SAME / _FP8_E4M3 (fused step only)            */
    int reserved0;     /* must be zero                                              */
    float* k_scale;    /* FP8: device fp32 scales of K; NVFP4: E4M3 block-scale bytes */
    float* v_scale;    /* the same for V (NULL for a same-dtype cache)               */
    float nvfp4_k_global; /* NVFP4: per-tensor scale g of K (0 = 1; else must be 0)   */
    float nvfp4_v_global; /* NVFP4: per-tensor scale g of V (0 = 1; else must be 0)   */
    int reserved[2];   /* must be zero                                              */
} rope3d_options;

/* Opaque frequency configuration: split, theta, schedule, the fp32 inverse
 * frequencies and, optionally, per-axis cos/sin tables in device memory. */
typedef struct rope3d_tables rope3d_tables;

/*
 * Build the frequency configuration on the current device ("RoPE Frequency
 * Precomputation", Section 3.4.1 item 2: contiguous precomputed tensors instead of
 * a per-call cache).  For each axis a in (t, h, w) and each position p < max_a the
 * table holds cos and sin of p * inv_a[j] computed in fp64 and stored as fp32,
 * laid out [max_a][n_a] of (cos, sin) pairs.  max_t = max_h = max_w = 0 builds no
 * tables: only ROPE3D_TRIG_ONTHEFLY can then be used.
 *   out       : receives the handle (set to NULL on failure)
 *   head_dim  : must equal 2 (n_t + n_h + n_w); the kernels support 128
 *   theta     : base, > 1 (10000 for the Wan2.1-style backbone)
 *   schedule  : ROPE3D_SCHEDULE_*
 *   cuda_stream: stream for the table upload; the call synchronises it before
 *               returning (this is set-up, not the per-chunk path)
 * Errors: EINVAL for bad sizes, ECUDA if allocation or upload fails, EDEVICE if the
 * current device is not compute capability 10.0.  Ownership: the library; release
 * with rope3d_tables_destroy on the same device.
 */
ROPE3D_API int rope3d_tables_init(rope3d_tables** out, int head_dim, int n_t, int n_h, int n_w,
                       double theta, int max_t, int max_h, int max_w, int schedule,
                       void* cuda_stream);

/* Free the tables (NULL is accepted).  Synchronises the device that holds them. */
ROPE3D_API void rope3d_tables_destroy(rope3d_tables* tables);

/*
 * The fused step for one token range of one chunk (Algorithm 3 steps 2, 3 and 5 on
 * a rank whose slice begins at Delta = token_begin, Section 3.3.3), for all B
 * samples, which share grid, start frame and slot:
 *   q_out[b][r]           = RoPE(RMSNorm(q[b][r]; q_norm_w, eps), pos(i))
 *   k_cache[b][row(i)]    = RoPE(RMSNorm(k[b][r]; k_norm_w, eps), pos(i))
 *   v_cache[b][row(i)]    = v[b][r]                       (bit copy)
 * with i = token_begin + r, pos(i) the decode above with s = frame_offset, and
 * row(i) = (slot + i) mod cache_tokens.  Arithmetic is fp32; bf16 results are
 * rounded once, to nearest even, when stored.
 *   q, k, v   : [B][n_tok][N][D] of dtype (device, read only)
 *   q_out     : [B][n_tok][N][D]; may be q itself (in place), must not overlap k, v
 *               or the caches otherwise
 *   B, N, D   : batch, heads, head size (D = 128)
 *   dtype     : ROPE3D_F32 or ROPE3D_BF16
 *   token_begin, token_end : 0 <= begin < end <= T*H*W; end - begin <= cache_tokens
 *   frame_offset : start frame s >= 0 of the chunk (Self-Forcing's start_frame)
 *   T, H, W   : the chunk's latent grid (frames, rows, columns), each >= 1
 *   q_norm_w, k_norm_w : [N*D] fp32 RMSNorm weights (device)
 *   eps       : >= 0, added to the mean square
 *   k_cache, v_cache : [B][cache_tokens][N][D] of dtype; only the rows of this range
 *               are written; they must not overlap each other or any input
 *   cache_tokens, slot : cache rows (>= 1) and slot >= 0 of global index 0
 *   tables    : from rope3d_tables_init on this device, with D = its head_dim
 *   trig      : ROPE3D_TRIG_TABLE (needs s + floor((token_end-1)/(H W)) < max_t,
 *               H <= max_h, W <= max_w) or ROPE3D_TRIG_ONTHEFLY
 * Errors: EINVAL, ERANGE, EALIGN, EOVERLAP, EDEVICE, ECUDA as above.
 */
ROPE3D_API int rope3d_qk_norm_rope_append(const void* q, const void* k, const void* v, void* q_out,
                               int64_t B, int64_t N, int D, int dtype,
                               int64_t token_begin, int64_t token_end, int64_t frame_offset,
                               int T, int H, int W,
                               const float* q_norm_w, const float* k_norm_w, float eps,
                               void* k_cache, void* v_cache, int64_t cache_tokens,
                               int64_t slot, const rope3d_tables* tables, int trig,
                               void* cuda_stream);

/*
 * rope3d_qk_norm_rope_append with options (pairing and cache layout; see
 * rope3d_options).  With ROPE3D_CACHE_HEAD_MAJOR the caches are [B][N][cache_tokens][D]
 * and head n of token i goes to k_cache[b][n][(slot + i) mod cache_tokens].  Errors as
 * for rope3d_qk_norm_rope_append, plus EINVAL for unknown option values.
 */
ROPE3D_API int rope3d_qk_norm_rope_append_ex(
    const void* q, const void* k, const void* v, void* q_out, int64_t B, int64_t N, int D,
    int dtype, int64_t token_begin, int64_t token_end, int64_t frame_offset, int T, int H, int W,
    const float* q_norm_w, const float* k_norm_w, float eps, void* k_cache, void* v_cache,
    int64_t cache_tokens, int64_t slot, const rope3d_tables* tables, int trig,
    const rope3d_options* options, void* cuda_stream);

/*
 * Sequence-parallel step with the all-to-all folded in: Algorithm 3 steps 3-5 ("Causal-RoPE
 * SP", Section 3.3.3; the FusedAllToAll of Section 3.4.1 item 1 with scatter over heads and
 * gather over the sequence).  This rank holds q, k, v for its own token range
 * [token_begin, token_end) with all N heads (layout as for rope3d_qk_norm_rope_append).  The
 * heads are split evenly over dest->ranks = P ranks: rank r owns heads
 * [r N/P, (r+1) N/P).  For every token i of the range and head n the step computes the same
 * values as rope3d_qk_norm_rope_append and stores them at the owner r of n, local head
 * n' = n - r N/P:
 *   q:  dest->q[r]        [B][dest->q_rows][N/P][D], row i - dest->q_row0 (the owner's
 *                          buffer holds the gathered sequence; usually q_row0 = 0 and
 *                          q_rows = T*H*W);
 *   K:  dest->k_cache[r]  [B][cache_tokens][N/P][D] (or [B][N/P][cache_tokens][D] with
 *                          options->cache_layout = ROPE3D_CACHE_HEAD_MAJOR), cache row
 *                          (slot + i) mod cache_tokens;
 *   V:  dest->v_cache[r]  likewise, a bit copy.
 * Run on every rank with its own range and the same dest tables (each rank listing the
 * ranks' buffers in rank order), the ranks together produce the whole-sequence result
 * split by heads, bit-identical to rope3d_qk_norm_rope_append on the whole sequence.
 *
 * Destination pointers are device addresses valid on the calling device: this device's
 * memory, or another GPU's memory mapped into this process (CUDA IPC, or a symmetric-memory
 * mapping); stores to another GPU go over NVLink as plain peer stores.  The call does not
 * synchronise with the other ranks: before a rank reads what others wrote, every rank's
 * step must have completed (for example a stream synchronisation followed by a barrier of
 * the process group).  Options: adjacent pairing and same-dtype caches only
 * (ROPE3D_EINVAL otherwise); the cache layout option applies.  Errors: P outside
 * [1, ROPE3D_SP_MAX_RANKS] or N not divisible by P (EINVAL); the token range outside
 * [q_row0, q_row0 + q_rows) (ERANGE); a NULL or misaligned destination (EINVAL / EALIGN);
 * destinations that overlap one another or an input, as far as their address ranges show
 * it (EOVERLAP).  Other arguments and errors as for rope3d_qk_norm_rope_append.
 */
#define ROPE3D_SP_MAX_RANKS 8

typedef struct rope3d_sp_dest {
    int ranks;                               /* P                                      */
    int reserved0;                           /* must be zero                           */
    int64_t q_rows;                          /* rows per sample of each q buffer       */
    int64_t q_row0;                          /* global token index of q row 0          */
    void* q[ROPE3D_SP_MAX_RANKS];            /* rank r's q buffer (entries >= P unused) */
    void* k_cache[ROPE3D_SP_MAX_RANKS];      /* rank r's K cache                       */
    void* v_cache[ROPE3D_SP_MAX_RANKS];      /* rank r's V cache                       */
} rope3d_sp_dest;

ROPE3D_API int rope3d_qk_norm_rope_append_sp(
    const void* q, const void* k, const void* v, int64_t B, int64_t N, int D, int dtype,
    int64_t token_begin, int64_t token_end, int64_t frame_offset, int T, int H, int W,
    const float* q_norm_w, const float* k_norm_w, float eps, const rope3d_sp_dest* dest,
    int64_t cache_tokens, int64_t slot, const rope3d_tables* tables, int trig,
    const rope3d_options* options, void* cuda_stream);

/*
 * The all-to-all after attention, Algorithm 3's last step (o <- AllToAll(o,
 * scatter_dim=1, gather_dim=2)): the inverse exchange of the head scatter above.  Rank
 * dest->rank = r holds o [B][L][heads_per_rank][D] -- the whole sequence of L tokens for
 * its own heads [r hl, (r+1) hl), hl = heads_per_rank -- and stores every token i to the
 * rank r' whose slice [dest->cuts[r'], dest->cuts[r'+1]) contains i, as that rank's rows
 * with all N = P hl heads:
 *   dest->out[r'] [B][cuts[r'+1] - cuts[r']][N][D], row i - cuts[r'], heads
 *   [r hl, (r+1) hl) of that row.
 * Run on every rank with the same cuts and out tables (each listing the ranks' buffers in
 * rank order), the ranks together leave in rank r' its token slice with every head.  A
 * bit copy: o and every out[r'] must be 16-byte aligned; when all of them are 32-byte
 * aligned the copy moves 32-byte units, otherwise 16-byte ones.  Destinations
 * are device addresses valid on the calling device (this device's memory, or another
 * GPU's memory mapped into this process); stores to another GPU are plain peer stores over
 * NVLink.  The call does not synchronise with the other ranks (as for the head scatter).
 * Errors: dest->ranks outside [1, ROPE3D_SP_MAX_RANKS] or rank outside [0, P) (EINVAL);
 * cuts not rising from 0 to L (ERANGE); D != 128, an unknown dtype, a NULL o or a NULL
 * out[r'] whose slice is not empty (EINVAL); a misaligned pointer (EALIGN); outputs that
 * overlap one another or o (EOVERLAP).
 */
typedef struct rope3d_sp_out_dest {
    int ranks;                               /* P                                      */
    int rank;                                /* this rank r, 0 <= r < P                */
    int64_t cuts[ROPE3D_SP_MAX_RANKS + 1];   /* rank r' holds tokens [cuts[r'], cuts[r'+1]) */
    void* out[ROPE3D_SP_MAX_RANKS];          /* rank r's output buffer (entries >= P unused) */
} rope3d_sp_out_dest;

ROPE3D_API int rope3d_sp_output_all_to_all(const void* o, int64_t B, int64_t L,
                                           int64_t heads_per_rank, int D, int dtype,
                                           const rope3d_sp_out_dest* dest, void* cuda_stream);

/*
 * The QKV projection that feeds the step (Algorithm 1/3 step 1, "q, k, v <- QKV(x)"; the
 * paper fuses it with the rotary step, Section 3.4.1 item 3), on the tensor cores:
 * y = x W^T + b with x [M][K] bf16 (token rows), w_qkv [3 N D][K] bf16 (an nn.Linear
 * weight: the q rows, then the k rows, then the v rows) and b_qkv [3 N D] fp32 (NULL: no
 * bias); fp32 accumulation, one round to nearest even to bf16.  The q, k and v column
 * blocks of y go to q_out, k_out, v_out, each [M][N][D] bf16.  K must be a multiple of
 * 64; x and w_qkv 16-byte aligned.  The kernel holds all of each SM's tensor memory while
 * it runs: calls on concurrent streams serialise on it.  The caller owns every buffer; the
 * call allocates nothing.  Its pipeline waits are bounded (2 s each); a launch that gives
 * up leaves its outputs incomplete and, having no tables, reports nothing.  Errors: NULL
 * pointers, D != 128, N < 1, M < 1, or K not a multiple of 64 or above 2^20 (EINVAL);
 * M > 2^30 or 3 N D > 2^24 (ERANGE); misaligned pointers, a bias not 4-byte aligned
 * (EALIGN); outputs that overlap x, w_qkv or one another (EOVERLAP); EDEVICE, ECUDA.
 */
ROPE3D_API int rope3d_qkv_project(const void* x, const void* w_qkv, const float* b_qkv, int64_t M,
                                  int64_t K, int64_t N, int D, void* q_out, void* k_out,
                                  void* v_out, void* cuda_stream);

/*
 * The projection and the step in one call: x [B][n_tok][K] bf16 holds the token rows of
 * [token_begin, token_end); q, k, v = QKV(x) as in rope3d_qkv_project (fp32 accumulation),
 * then the step of rope3d_qk_norm_rope_append on them, with V stored straight into the V
 * cache at each token's cache row by the projection's epilogue.
 *   - When N D is a multiple of 256 (even head counts) the projection's epilogue applies
 *     the RMSNorm weight and the rotation to the fp32 q and k tiles, stores them to q_out
 *     and the K cache, and records each row's partial sum of squares per tile in the
 *     workspace; a light second kernel then scales every q and K row by
 *     1 / sqrt(mean(x^2) + eps) in place (a fixed-order sum, so results do not depend on
 *     scheduling or on slicing).  The normalisation uses the fp32 projections, and q, K
 *     are rounded to bf16 twice (before and after the scale).
 *   - Otherwise the projection rounds q and k to bf16 (q into q_out, k into the workspace)
 *     and the step then normalises and rotates them (V already in the cache).
 * workspace: device scratch of rope3d_qkv_workspace_bytes(B, n_tok, N, D) bytes (no
 * initialisation needed; 0 is returned for invalid sizes).  bf16 only; options: the cache
 * layout (adjacent pairing, bf16 caches; EINVAL otherwise).  A workspace smaller than
 * needed is EINVAL; q_out, the workspace and the caches must not overlap one another, x
 * or w_qkv (EOVERLAP).  A wait that gives up is recorded in the tables' status word
 * (rope3d_check_device_status).  Other arguments and errors as for
 * rope3d_qk_norm_rope_append and rope3d_qkv_project.
 */
ROPE3D_API size_t rope3d_qkv_workspace_bytes(int64_t B, int64_t n_tok, int64_t N, int D);

ROPE3D_API int rope3d_qkv_norm_rope_append(
    const void* x, const void* w_qkv, const float* b_qkv, int64_t K, int64_t B, int64_t N, int D,
    int64_t token_begin, int64_t token_end, int64_t frame_offset, int T, int H, int W,
    const float* q_norm_w, const float* k_norm_w, float eps, void* q_out, void* workspace,
    size_t workspace_bytes, void* k_cache, void* v_cache, int64_t cache_tokens, int64_t slot,
    const rope3d_tables* tables, int trig, const rope3d_options* options, void* cuda_stream);

/*
 * The rotation alone -- CausalRoPE of Algorithm 3 step 3 / Algorithm 2 -- on one
 * token range: out[b][r] = RoPE(x[b][r], pos(token_begin + r)).  x and out are
 * [B][n_tok][N][D] of dtype; out may be x (in place) or must not overlap it.  Other
 * arguments as for rope3d_qk_norm_rope_append.
 */
ROPE3D_API int rope3d_apply(const void* x, void* out, int64_t B, int64_t N, int D, int dtype,
                 int64_t token_begin, int64_t token_end, int64_t frame_offset,
                 int T, int H, int W, const rope3d_tables* tables, int trig,
                 void* cuda_stream);

/* rope3d_apply with options (only the pairing applies). */
ROPE3D_API int rope3d_apply_ex(const void* x, void* out, int64_t B, int64_t N, int D, int dtype,
                               int64_t token_begin, int64_t token_end, int64_t frame_offset,
                               int T, int H, int W, const rope3d_tables* tables, int trig,
                               const rope3d_options* options, void* cuda_stream);

/*
 * Integer part of the step, for inspection: for each index i of [token_begin,
 * token_end) writes out[4 (i - token_begin) + {0,1,2,3}] = t_g, h, w and the cache
 * row (slot + i) mod cache_tokens, as int64 into the device array out
 * ([n_tok][4], 8-byte aligned).  Section 3.3.3; Algorithm 3, step 3.
 */
ROPE3D_API int rope3d_decode_positions(int64_t token_begin, int64_t token_end, int64_t frame_offset,
                            int T, int H, int W, int64_t cache_tokens, int64_t slot,
                            int64_t* out, void* cuda_stream);

/*
 * Device-side status of the kernels launched with these tables.  The fused kernel that
 * streams rows through shared memory waits on each stage with a time limit (2 s); if a
 * stage never fills, the kernel stops, its output rows are incomplete, and it records
 * the event in a device word that belongs to the tables.  This call synchronises
 * cuda_stream, reads and clears that word, and returns ROPE3D_ETIMEOUT if any launch
 * since the last check gave up, else ROPE3D_OK (ECUDA / EDEVICE / EINVAL on failure to
 * read it).  Not needed on the normal path; intended for health checks.
 *
 * A library built with -DROPE3D_DEVICE_CHECKS (rotary_position_encoding_b200.build
 * --checked, librope3d_checked.so) also tests, in the step kernels, every cache row,
 * table row and sequence-parallel destination q row it derives against the extents of
 * the call.  A token row whose cache row (or destination q row) lies outside is not
 * stored at all; a table row outside its table is not read (cos and sin are taken as 1
 * and 0).  Either is recorded in the same word, which this call then reports as
 * ROPE3D_EINDEX.  The host checks of
 * every entry point make that unreachable for valid arguments; the checked build guards
 * the kernels' own index arithmetic.  No kernel traps in either build.
 */
ROPE3D_API int rope3d_check_device_status(const rope3d_tables* tables, void* cuda_stream);

/*
 * The fused step without any device allocation.  The paper has no counterpart; this
 * entry point exists for callers that cannot call cudaMalloc: a host framework that owns
 * all device memory through its own allocator and forbids direct allocations, a process
 * whose caching allocator already holds the free device memory, or a latency-critical
 * loop that cannot afford cudaMalloc's implicit synchronisation.  rope3d_tables_init
 * allocates (its cos/sin tables and a status word), so those callers cannot use it.
 *
 * Here the frequency configuration is passed directly (n_t + n_h + n_w = 64, theta,
 * schedule), and everything the step needs beyond the caller's inputs and outputs sits
 * in one file-scope device array of 65,792 bytes that every GPU loading this library
 * holds until the process exits: a status word and room for 8192 (cos, sin) entries.
 * With trig = ROPE3D_TRIG_TABLE each call computes, in fp64 on the host, the cos/sin rows
 * of its own positions -- (frames touched) * n_t + H * n_h + W * n_w entries -- and
 * copies them into that array with cudaMemcpyAsync on cuda_stream, ahead of the call's
 * kernel in stream order.  The rows come from a library-owned pageable host buffer: the
 * runtime has taken them (staged or copied) when the copy call returns, and the library
 * holds a lock from the rows' computation until then, so a later call cannot overwrite
 * them.  Nothing here waits for cuda_stream to drain; the runtime may do so for a
 * pageable copy.  A call needing more than 8192 entries returns ROPE3D_ERANGE and
 * launches nothing.  With ROPE3D_TRIG_ONTHEFLY nothing is copied.  Each call first
 * clears the status word.  Outputs are bit-identical to
 * rope3d_qk_norm_rope_append with tables built from the same configuration.
 *
 * Every call shares the array and it keeps the last call's contents; calls that overlap
 * on the GPU (on different streams or from different host threads) race on it and must
 * be serialised by the caller.  The status word of the bounded waits is read back by
 * rope3d_noalloc_check_status.  The first call on a device looks up the array's device
 * address (one-time set-up with that device current).  Other arguments, layouts and
 * errors are those of rope3d_qk_norm_rope_append.
 */
ROPE3D_API int rope3d_qk_norm_rope_append_noalloc(
    const void* q, const void* k, const void* v, void* q_out, int64_t B, int64_t N, int D,
    int dtype, int64_t token_begin, int64_t token_end, int64_t frame_offset, int T, int H, int W,
    const float* q_norm_w, const float* k_norm_w, float eps, void* k_cache, void* v_cache,
    int64_t cache_tokens, int64_t slot, int n_t, int n_h, int n_w, double theta, int schedule,
    int trig, void* cuda_stream);

/*
 * The status word of rope3d_qk_norm_rope_append_noalloc on the current device, read and
 * cleared as rope3d_check_device_status does for a tables object: synchronises
 * cuda_stream, copies the word (a 4-byte device-to-host copy into the caller's stack; no
 * allocation), clears it when it is set, and returns ROPE3D_OK, ROPE3D_ETIMEOUT (a
 * bounded wait of the last no-allocation call gave up; its outputs are incomplete) or
 * ROPE3D_EINDEX (checked build only).  The word is the one every no-allocation call
 * clears first, so it reports the calls since the last read or the last call, whichever
 * came later.  ROPE3D_ECUDA if the copy fails.
 */
ROPE3D_API int rope3d_noalloc_check_status(void* cuda_stream);

/* Fixed text for a status code (never NULL). */
ROPE3D_API const char* rope3d_strerror(int status);

/* Details of the calling thread's most recent failure ("" if none). */
ROPE3D_API const char* rope3d_last_error(void);

/* Library version as major * 10000 + minor * 100 + patch. */
ROPE3D_API int rope3d_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ROPE3D_H */
