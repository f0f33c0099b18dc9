// rope3d_kernels.cuh -- sm_100a kernels of the fused QK-RMSNorm + causal 3D RoPE +
// KV-cache append step ("Accelerating Video Generation Inference with Sequential-
// Parallel 3D Positional Encoding Using a Global Time Index", Yuan & Li: Sections
// 3.3.1-3.3.3, Algorithm 2, Algorithm 3 steps 3 and 5).
//
// The step moves 6 * N * 128 elements per token and does ~15 flops per element of
// q and k, so it is bound by HBM bandwidth, not by arithmetic: no tensor cores.
//
// Shared design of both fused kernels:
//   * A "team" of TPR threads (a multiple of 32) owns one token row at a time.
//     Thread t of a team holds the 16-byte vectors t, t + TPR, t + 2 TPR, ... of the
//     row.  TPR is a multiple of the vectors per head, so a thread always sees the
//     same position inside a head, hence the same few complex pairs: its cos/sin are
//     computed once per row and reused for every head it holds and for q and k.
//   * RMSNorm needs the sum of squares of the whole N*128 row before any output, so
//     a thread keeps its vectors of the row in registers; the sum is a fixed warp
//     butterfly followed, for multi-warp teams, by a fixed-order sum of the warps'
//     partials (one named barrier per row, double-buffered partials).  The reduction
//     order depends only on N and the dtype, never on the token range or the grid,
//     so any slice of a sequence is bit-identical to the whole.
//   * Blocks are persistent; each block stages the two RMSNorm weight vectors in
//     shared memory once, and its teams stride over the (batch, token) rows.
//
// qk_norm_rope_kernel reads the rows straight into registers (coalesced 128-bit
// loads), so the bytes in flight per SM are bounded by the register file.
// qk_norm_rope_tma_kernel (rope3d_tma.cuh) streams rows into a ring of shared-memory
// stages with bulk asynchronous copies, decoupling bytes in flight from registers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rope3d {

constexpr int kHeadDim = 128;
constexpr int kPairs = kHeadDim / 2;
constexpr int kMaxTeamsPerBlock = 15;  // named barriers 1..15 (0 is __syncthreads)
constexpr int kMaxBlockThreads = 512;  // leaves up to 128 registers per thread
constexpr int kTmaMaxBlockThreads = 320;  // ring kernel: one block per SM, up to 204 registers

// kModeFusedSP: the fused step with head-scatter stores (the sequence-parallel
// all-to-all folded into the step): each head goes to the destination rank that owns it.
// kModeFusedNoV: the fused step for q and K only (V was appended by the producer of q,
// k, v -- the QKV projection's epilogue).
enum Mode : int { kModeFused = 0, kModeApply = 1, kModeFusedSP = 2, kModeFusedNoV = 3 };
constexpr int kMaxRanks = 8;  // head-scatter destinations (one node)
// Checked build (-DROPE3D_DEVICE_CHECKS): the kernels test every cache row, table row
// and destination q row they derive against the extents the host passed, and on a
// mismatch record kStatusIndexRange in the status word and skip that access -- no trap.
// The host validates every argument before a launch, so in a correct build the checks
// never fire; they guard the index arithmetic itself.
#ifdef ROPE3D_DEVICE_CHECKS
constexpr bool kDeviceChecks = true;
#else
constexpr bool kDeviceChecks = false;
#endif
constexpr int kStatusIndexRange = 2;
// KV-cache element formats of the fused step
enum CacheFmt : int { kCacheSame = 0, kCacheFp8 = 1, kCacheNvfp4 = 2 };
enum Trig : int { kTrigTable = 0, kTrigOnTheFly = 1 };
// Pairing of a head's elements into complex pairs: adjacent (2j, 2j+1) -- the complex
// view of Wan2.1 -- or rotate_half (j, j + 64), the cos/sin form of M-RoPE.
enum Pairing : int { kPairAdjacent = 0, kPairHalf = 1 };

// Division of n < 2^31 by a fixed divisor d in [1, 2^31) without a divide instruction:
// q = floor(n m / 2^s) with l = ceil(log2 d), s = 31 + l and m = floor(2^s / d) + 1 < 2^32
// (the round-up method for dividends of 31 bits; m d = 2^s + e with 0 < e <= d, so the
// error term n e / (d 2^s) stays below 2^-l <= 1/d and the floor is exact).
struct FastDiv {
    uint32_t m;
    uint32_t s;
};

__host__ __device__ inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t l = 0;
    while (l < 31 && (1u << l) < d) ++l;
    FastDiv f;
    f.s = 31 + l;
    f.m = (uint32_t)((1ull << f.s) / d + 1);
    return f;
}

__host__ __device__ __forceinline__ uint32_t fast_div(uint32_t n, FastDiv f) {
    return (uint32_t)(((uint64_t)n * f.m) >> f.s);
}

struct Params {
    const void* q;        // fused: q;  apply: x
    const void* k;
    const void* v;
    void* q_out;          // fused: q_out;  apply: out
    void* k_cache;
    void* v_cache;
    const float* q_w;     // [dim] RMSNorm weights
    const float* k_w;
    const float2* tab_t;  // [max_t][n_t] (cos, sin)
    const float2* tab_h;  // [max_h][n_h]
    const float2* tab_w;  // [max_w][n_w]
    int* status;          // device status word of the bounded waits (TMA kernel)
    int64_t n_tok;        // rows per batch sample
    int64_t units;        // B * n_tok rows in total
    int64_t token_begin;
    int64_t frame_offset;
    int64_t cache_tokens;
    int64_t slot;
    int64_t hw;           // H * W
    uint64_t wait_limit_ns;  // TMA kernel: give up on a stage after this long
    int H;
    int W;
    int dim;              // N * 128 elements per row
    int dim_vecs;         // 16-byte vectors per row
    int tpr;              // threads per team (multiple of 32)
    int teams;            // teams per block
    int small_idx;        // all index arithmetic fits in 32 bits
    FastDiv div_ntok, div_hw, div_w, div_cache;  // for the 32-bit decode
    float eps;
    float inv_dim;        // 1 / dim
    int n_t, n_h, n_w;
    // TMA kernel shared-memory layout (byte offsets into dynamic shared memory)
    int stages;           // ring stages per team
    uint32_t row_bytes;   // bytes of one token row of one tensor
    uint32_t tx_extra;    // extra bytes each stage waits for (0; tests use it to time out)
    uint32_t off_bars, off_fail, off_part, off_w, off_stage;
    // layout options
    int cache_head_major;  // caches are [B][N][cache_tokens][D] instead of [B][cache_tokens][N][D]
    int n_heads;           // N
    int vph_log2;          // log2 of the 16-byte vectors per head
    float* k_scale;        // FP8 caches: per (token, head) scales, laid out like the cache rows
    float* v_scale;
    uint8_t* k_bscale;     // NVFP4 caches: E4M3 scale per 16-element block, laid out like the rows
    uint8_t* v_bscale;
    float k_global, v_global;  // NVFP4 per-tensor scales g
    float k_inv6g, v_inv6g;    // fp32(1 / fp32(6 g))
    // head-scatter destinations (kModeFusedSP): rank r owns heads [r*sp_heads, (r+1)*sp_heads)
    int sp_ranks;
    int sp_heads;          // heads per rank
    int64_t sp_q_rows;     // rows per batch sample of a destination q buffer
    int64_t sp_q_row0;     // global token index held by a destination q buffer's row 0
    void* sp_dst[3 * kMaxRanks];  // rank r: q [B][sp_q_rows][sp_heads][D], k and v caches
    int64_t tab_rows_t;      // rows of the t, h and w tables (read by the checked build)
    int tab_rows_h, tab_rows_w;
    int64_t check_shrink;    // checked build, tests only: cache rows the row check withholds
    float inv_freq[kPairs];  // fp32 angle per unit position of every pair
};

// ---------------------------------------------------------------- element types

template <typename T> struct VecTraits;

template <> struct VecTraits<__nv_bfloat16> {
    using Vec = uint4;                 // 8 bf16 = 4 complex pairs, one pair per 32-bit word
    static constexpr int kPairsPerVec = 4;
    static constexpr int kVecsPerHead = kHeadDim / 8;
    __device__ static inline void pair(const Vec& x, int m, float& re, float& im) {
        uint32_t u = m == 0 ? x.x : m == 1 ? x.y : m == 2 ? x.z : x.w;
        re = __uint_as_float(u << 16);           // element 2j (lower address)
        im = __uint_as_float(u & 0xffff0000u);   // element 2j + 1
    }
    __device__ static inline void set_pair(Vec& x, int m, float re, float im) {
        __nv_bfloat162 h = __floats2bfloat162_rn(re, im);  // round to nearest even
        uint32_t u = *reinterpret_cast<uint32_t*>(&h);
        if (m == 0) x.x = u; else if (m == 1) x.y = u; else if (m == 2) x.z = u; else x.w = u;
    }
    static constexpr int kElems = 8;
    __device__ static inline float elem(const Vec& x, int m) {
        const uint32_t u = (m >> 1) == 0 ? x.x : (m >> 1) == 1 ? x.y : (m >> 1) == 2 ? x.z : x.w;
        return (m & 1) ? __uint_as_float(u & 0xffff0000u) : __uint_as_float(u << 16);
    }
    __device__ static inline Vec pack_elems(const float (&v)[8]) {
        Vec o;
#pragma unroll
        for (int w = 0; w < 4; ++w) set_pair(o, w, v[2 * w], v[2 * w + 1]);
        return o;
    }
};

template <> struct VecTraits<float> {
    using Vec = float4;                // 4 floats = 2 complex pairs
    static constexpr int kPairsPerVec = 2;
    static constexpr int kVecsPerHead = kHeadDim / 4;
    __device__ static inline void pair(const Vec& x, int m, float& re, float& im) {
        re = m == 0 ? x.x : x.z;
        im = m == 0 ? x.y : x.w;
    }
    __device__ static inline void set_pair(Vec& x, int m, float re, float im) {
        if (m == 0) { x.x = re; x.y = im; } else { x.z = re; x.w = im; }
    }
    static constexpr int kElems = 4;
    __device__ static inline float elem(const Vec& x, int m) {
        return m == 0 ? x.x : m == 1 ? x.y : m == 2 ? x.z : x.w;
    }
    __device__ static inline Vec pack_elems(const float (&v)[4]) {
        return make_float4(v[0], v[1], v[2], v[3]);
    }
};

// Pairs a thread rotates: with adjacent pairing the kPairsPerVec pairs of its vector;
// with rotate_half the kElems pairs whose real (first half of the head) or imaginary
// (second half) parts its vector holds.
template <typename T, int PAIR>
struct PairCount {
    static constexpr int value =
        PAIR == kPairAdjacent ? VecTraits<T>::kPairsPerVec : VecTraits<T>::kElems;
};

// Vector (16-byte unit of the row) that slot s of thread t holds.
//  adjacent pairing: t + s * TPR -- coalesced, and a thread's position inside a head
//                    is t mod (vectors per head);
//  rotate_half:      slots come in twos over "half units" u = t + (s/2) * TPR; unit u
//                    is position u mod HALF of head u / HALF, and its even slot holds
//                    the head's first-half vector there, its odd slot the second-half
//                    vector HALF further on -- the real and imaginary parts of the same
//                    pairs, so no data crosses lanes.
// In both, a vector index >= dim_vecs marks an empty slot.
template <typename T, int PAIR>
__device__ __forceinline__ int slot_vec(int t, int s, int tpr) {
    using Tr = VecTraits<T>;
    if (PAIR == kPairAdjacent) return t + s * tpr;
    constexpr int HALF = Tr::kVecsPerHead / 2;
    const int u = t + (s >> 1) * tpr;
    return (u / HALF) * Tr::kVecsPerHead + (u % HALF) + (s & 1) * HALF;
}

// First pair of a thread whose vectors sit at position `pos_in_head` of their heads.
template <typename T, int PAIR>
__device__ __forceinline__ int first_pair(int pos_in_head) {
    using Tr = VecTraits<T>;
    return PAIR == kPairAdjacent ? pos_in_head * Tr::kPairsPerVec
                                 : (pos_in_head % (Tr::kVecsPerHead / 2)) * Tr::kElems;
}

// ---------------------------------------------------------------- memory helpers

__device__ __forceinline__ uint4 load_stream(const uint4* p) { return __ldcs(p); }
__device__ __forceinline__ float4 load_stream(const float4* p) { return __ldcs(p); }
// Outputs are written once and not read again by this kernel: streaming (evict-first)
// stores keep them from displacing lines still in use (measured 1-2% faster on B200).
__device__ __forceinline__ void store_out(uint4* p, const uint4& v) { __stcs(p, v); }
__device__ __forceinline__ void store_out(float4* p, const float4& v) { __stcs(p, v); }

// Programmatic dependent launch: let the next kernel on the stream start its prologue
// while this grid drains, and wait for the previous grid (and its memory) before this
// grid reads anything from global memory.  Both are no-ops without the launch attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_previous_grid() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void team_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float warp_allreduce_sum(float x) {
    // Butterfly: every lane ends with the bitwise-same total (each step adds the same
    // two operands, only their order differs, and fp addition is commutative).
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// ---------------------------------------------------------------- per-row pieces

// Position of token row u (Section 3.3.3: i = token_begin + r, t_g = s + floor(i/HW),
// h = floor(i/W) mod H, w = i mod W) and its rolling-cache row (slot + i) mod C.
struct RowPos {
    int64_t b, r, i, t_g, crow;
    int h, w;
    bool ok;  // checked build: the row's cache row and position lie inside their extents
};

__device__ __forceinline__ void record_index_error(const Params& p) {
    atomicOr(p.status, kStatusIndexRange);
}

__device__ __forceinline__ RowPos decode_row(const Params& p, int64_t u) {
    RowPos q;
    if (p.small_idx) {
        const uint32_t uu = (uint32_t)u, ntok = (uint32_t)p.n_tok;
        const uint32_t b = fast_div(uu, p.div_ntok);
        const uint32_t r = uu - b * ntok;
        const uint32_t i = (uint32_t)p.token_begin + r;
        const uint32_t hw = (uint32_t)p.hw, W = (uint32_t)p.W;
        const uint32_t tl = fast_div(i, p.div_hw);
        const uint32_t rem = i - tl * hw;
        const uint32_t h = fast_div(rem, p.div_w);
        q.b = b;
        q.r = r;
        q.i = i;
        q.t_g = p.frame_offset + tl;
        q.h = (int)h;
        q.w = (int)(rem - h * W);
        const uint32_t si = (uint32_t)p.slot + i;
        q.crow = si - fast_div(si, p.div_cache) * (uint32_t)p.cache_tokens;
    } else {
        q.b = u / p.n_tok;
        q.r = u - q.b * p.n_tok;
        q.i = p.token_begin + q.r;
        const int64_t tl = q.i / p.hw;
        const int64_t rem = q.i - tl * p.hw;
        q.h = (int)(rem / p.W);
        q.w = (int)(rem - (int64_t)q.h * p.W);
        q.t_g = p.frame_offset + tl;
        q.crow = (p.slot + q.i) % p.cache_tokens;
    }
    q.ok = true;
    if constexpr (kDeviceChecks) {
        q.ok = q.b < p.units / p.n_tok && q.r < p.n_tok && q.crow >= 0 &&
               q.crow < p.cache_tokens - p.check_shrink && q.h >= 0 && q.h < p.H &&
               q.w >= 0 && q.w < p.W;
        if (!q.ok) record_index_error(p);
    }
    return q;
}

// Index (in 16-byte vectors) of vector idx of a row's K/V in the cache, for the row's
// cache row: token-major [B][C][N][D] or head-major [B][N][C][D].
__device__ __forceinline__ int64_t cache_vec_index(const Params& p, const RowPos& pos, int idx) {
    if (!p.cache_head_major) return (pos.b * p.cache_tokens + pos.crow) * p.dim_vecs + idx;
    const int n = idx >> p.vph_log2;
    const int v = idx & ((1 << p.vph_log2) - 1);
    return (((pos.b * p.n_heads + n) * p.cache_tokens + pos.crow) << p.vph_log2) + v;
}

// Index of the scale of head n of a row's K/V in an FP8 cache's scale array:
// [B][C][N] (token-major) or [B][N][C] (head-major).
__device__ __forceinline__ int64_t cache_scale_index(const Params& p, const RowPos& pos, int n) {
    return p.cache_head_major ? (pos.b * p.n_heads + n) * p.cache_tokens + pos.crow
                              : (pos.b * p.cache_tokens + pos.crow) * p.n_heads + n;
}

// The complex pairs a thread rotates (fixed for the thread's whole life).
template <int PPV>
struct PairInfo {
    float inv[PPV];             // angle per unit position
    int axis[PPV];              // 0 = t, 1 = h, 2 = w
    const float2* tab[PPV];     // table column of the pair (row 0)
    int stride[PPV];            // table row length of the pair's axis
};

template <int PPV>
__device__ __forceinline__ PairInfo<PPV> pair_info(const Params& p, int pair0) {
    PairInfo<PPV> pi;
#pragma unroll
    for (int m = 0; m < PPV; ++m) {
        const int j = pair0 + m;
        pi.inv[m] = p.inv_freq[j];
        if (j < p.n_t) {
            pi.axis[m] = 0; pi.tab[m] = p.tab_t + j; pi.stride[m] = p.n_t;
        } else if (j < p.n_t + p.n_h) {
            pi.axis[m] = 1; pi.tab[m] = p.tab_h + (j - p.n_t); pi.stride[m] = p.n_h;
        } else {
            pi.axis[m] = 2; pi.tab[m] = p.tab_w + (j - p.n_t - p.n_h); pi.stride[m] = p.n_w;
        }
    }
    return pi;
}

// cos and sin of each of the thread's pairs at (t_g, h, w): Section 3.3.2 item 2,
// phi_j = t_g theta_T,j | h theta_H,j | w theta_W,j on the pair's own axis.
template <int TRIG, int PPV>
__device__ __forceinline__ void pair_trig(const Params& p, const PairInfo<PPV>& pi,
                                          const RowPos& pos, float (&cs)[PPV],
                                          float (&sn)[PPV]) {
#pragma unroll
    for (int m = 0; m < PPV; ++m) {
        const int64_t x = pi.axis[m] == 0 ? pos.t_g : (pi.axis[m] == 1 ? (int64_t)pos.h
                                                                        : (int64_t)pos.w);
        if (kDeviceChecks && TRIG == kTrigTable) {
            const int64_t rows = pi.axis[m] == 0 ? p.tab_rows_t
                                 : (pi.axis[m] == 1 ? p.tab_rows_h : p.tab_rows_w);
            if (x < 0 || x >= rows) {
                record_index_error(p);
                cs[m] = 1.0f;
                sn[m] = 0.0f;
                continue;
            }
        }
        if (TRIG == kTrigTable) {
            const float2 e = __ldg(pi.tab[m] + x * pi.stride[m]);
            cs[m] = e.x;
            sn[m] = e.y;
        } else {
            const float phi = (float)x * pi.inv[m];
            sincosf(phi, &sn[m], &cs[m]);
        }
    }
}

// The same table in a lean form for the register kernel, where registers decide how many
// blocks fit an SM: per pair only its column in its axis table and its axis (two bits),
// the three axis rows found once per row.  Same cos and sin as above.  Measured on B200:
// 8 registers fewer at 720P, the FP8 step 3% and the register path 1% faster; the ring
// kernel, which has registers to spare, keeps the per-pair pointers (0.8% faster).
template <int PPV>
struct PairCols {
    float inv[PPV];   // angle per unit position (on-the-fly trig only)
    int col[PPV];     // the pair's column in its axis table
    uint32_t axes;    // two bits per pair: 0 = t, 1 = h, 2 = w
};

template <int PPV>
__device__ __forceinline__ PairCols<PPV> pair_cols(const Params& p, int pair0) {
    PairCols<PPV> pc;
    pc.axes = 0;
#pragma unroll
    for (int m = 0; m < PPV; ++m) {
        const int j = pair0 + m;
        pc.inv[m] = p.inv_freq[j];
        const uint32_t a = j < p.n_t ? 0u : (j < p.n_t + p.n_h ? 1u : 2u);
        pc.col[m] = a == 0 ? j : (a == 1 ? j - p.n_t : j - p.n_t - p.n_h);
        pc.axes |= a << (2 * m);
    }
    return pc;
}

template <int TRIG, int PPV>
__device__ __forceinline__ void pair_trig(const Params& p, const PairCols<PPV>& pc,
                                          const RowPos& pos, float (&cs)[PPV],
                                          float (&sn)[PPV]) {
    if constexpr (TRIG == kTrigTable) {
        const float2* rt = p.tab_t + pos.t_g * p.n_t;
        const float2* rh = p.tab_h + (int64_t)pos.h * p.n_h;
        const float2* rw = p.tab_w + (int64_t)pos.w * p.n_w;
#pragma unroll
        for (int m = 0; m < PPV; ++m) {
            const uint32_t a = (pc.axes >> (2 * m)) & 3u;
            if (kDeviceChecks) {
                const int64_t x = a == 0 ? pos.t_g : (a == 1 ? (int64_t)pos.h : (int64_t)pos.w);
                const int64_t rows = a == 0 ? p.tab_rows_t
                                            : (a == 1 ? p.tab_rows_h : p.tab_rows_w);
                if (x < 0 || x >= rows) {
                    record_index_error(p);
                    cs[m] = 1.0f;
                    sn[m] = 0.0f;
                    continue;
                }
            }
            const float2 e = __ldg((a == 0 ? rt : (a == 1 ? rh : rw)) + pc.col[m]);
            cs[m] = e.x;
            sn[m] = e.y;
        }
    } else {
#pragma unroll
        for (int m = 0; m < PPV; ++m) {
            const uint32_t a = (pc.axes >> (2 * m)) & 3u;
            const int64_t x = a == 0 ? pos.t_g : (a == 1 ? (int64_t)pos.h : (int64_t)pos.w);
            const float phi = (float)x * pc.inv[m];
            sincosf(phi, &sn[m], &cs[m]);
        }
    }
}

// acc + lo^2 + hi^2 for the two bf16 halves of a 32-bit word (lo, the element at the lower
// address, first), without widening them: fma.rn.f32.bf16 multiplies two bf16 operands
// (the product of two 8-bit significands is exact in fp32) and adds an fp32 operand with
// one rounding -- the same result as fmaf on the widened values.
__device__ __forceinline__ float fma_squares_bf16x2(uint32_t u, float acc) {
    asm("{\n"
        "  .reg .b16 lo, hi;\n"
        "  mov.b32 {lo, hi}, %1;\n"
        "  fma.rn.f32.bf16 %0, lo, lo, %0;\n"
        "  fma.rn.f32.bf16 %0, hi, hi, %0;\n"
        "}"
        : "+f"(acc)
        : "r"(u));
    return acc;
}

// Adds the squares of one vector of q and one of k to (sq, sk), in element order.  Every
// kernel sums a thread's vectors with this in slot order, so the sums are bit-identical
// across kernels.
__device__ __forceinline__ void accumulate_squares(const uint4& xq, const uint4& xk, float& sq,
                                                   float& sk) {
    sq = fma_squares_bf16x2(xq.x, sq);
    sq = fma_squares_bf16x2(xq.y, sq);
    sq = fma_squares_bf16x2(xq.z, sq);
    sq = fma_squares_bf16x2(xq.w, sq);
    sk = fma_squares_bf16x2(xk.x, sk);
    sk = fma_squares_bf16x2(xk.y, sk);
    sk = fma_squares_bf16x2(xk.z, sk);
    sk = fma_squares_bf16x2(xk.w, sk);
}
__device__ __forceinline__ void accumulate_squares(const float4& xq, const float4& xk, float& sq,
                                                   float& sk) {
    sq = fmaf(xq.x, xq.x, sq);
    sq = fmaf(xq.y, xq.y, sq);
    sq = fmaf(xq.z, xq.z, sq);
    sq = fmaf(xq.w, xq.w, sq);
    sk = fmaf(xk.x, xk.x, sk);
    sk = fmaf(xk.y, xk.y, sk);
    sk = fmaf(xk.z, xk.z, sk);
    sk = fmaf(xk.w, xk.w, sk);
}

// Sum of squares of this thread's share of one row of q and of k (fixed order).
template <typename T, int VPT, int PAIR>
__device__ __forceinline__ void partial_sum_squares(const typename VecTraits<T>::Vec (&xq)[VPT],
                                                    const typename VecTraits<T>::Vec (&xk)[VPT],
                                                    int t, int tpr, int dim_vecs, float& sq,
                                                    float& sk) {
    sq = 0.f;
    sk = 0.f;
#pragma unroll
    for (int s = 0; s < VPT; ++s)
        if (slot_vec<T, PAIR>(t, s, tpr) < dim_vecs) accumulate_squares(xq[s], xk[s], sq, sk);
}

// Team-wide totals of (sq, sk): warp butterfly, then the warps' partials in warp order.
// For multi-warp teams this is the row's one named barrier; it also orders every read
// of the row made before it ahead of everything after it.
__device__ __forceinline__ float2 team_sum(float sq, float sk, float2* s_part, int team,
                                           int teams, int warp_in_team, int warps_per_team,
                                           int lane, int tpr, int& parity) {
    sq = warp_allreduce_sum(sq);
    sk = warp_allreduce_sum(sk);
    if (warps_per_team > 1) {
        float2* part = s_part + (parity * teams + team) * warps_per_team;
        if (lane == 0) part[warp_in_team] = make_float2(sq, sk);
        team_barrier(1 + team, tpr);
        sq = 0.f;
        sk = 0.f;
        for (int wi = 0; wi < warps_per_team; ++wi) {
            const float2 pp = part[wi];
            sq += pp.x;
            sk += pp.y;
        }
        parity ^= 1;
    }
    return make_float2(sq, sk);
}

// The norm weights sit in shared memory permuted inside every group of four elements --
// (w0, w2, w1, w3) -- so that one 16-byte read gives the weights of the real parts of two
// neighbouring pairs and, as the other half, those of their imaginary parts: the operand
// layout of the packed fp32x2 arithmetic below.  Weights of elements e .. e + 3 (e a
// multiple of 4) in element order:
__device__ __forceinline__ float4 weights4(const float* s_w, int e) {
    const float4 a = *reinterpret_cast<const float4*>(s_w + e);
    return make_float4(a.x, a.z, a.y, a.w);
}

// A row's rotation for the thread's pairs, scaled by the row's RMSNorm factor rs, as
// fp32x2 lanes (pairs 2h and 2h + 1): c = rs cos, s = rs sin, ns = -(rs sin).
template <int PPV>
struct RowRot {
    float2 c[PPV / 2], s[PPV / 2], ns[PPV / 2];
};

template <int PPV>
__device__ __forceinline__ RowRot<PPV> row_rot(float rs, const float (&cs)[PPV],
                                               const float (&sn)[PPV]) {
    RowRot<PPV> r;
    const float2 p = make_float2(rs, rs), n = make_float2(-rs, -rs);
#pragma unroll
    for (int h = 0; h < PPV / 2; ++h) {
        const float2 c = make_float2(cs[2 * h], cs[2 * h + 1]);
        const float2 sv = make_float2(sn[2 * h], sn[2 * h + 1]);
        r.c[h] = __fmul2_rn(c, p);
        r.s[h] = __fmul2_rn(sv, p);
        r.ns[h] = __fmul2_rn(sv, n);
    }
    return r;
}

// RMSNorm and RoPE of one vector: y = x w (the weight), then (y_re + i y_im) times
// rs (cos + i sin) -- the row's 1/rms folded into the rotation -- two pairs per packed
// fp32x2 operation; the result as fp32 in element order.
template <typename T>
__device__ __forceinline__ void norm_rotate_f(
    const typename VecTraits<T>::Vec& x, const float* s_w, int e0,
    const RowRot<VecTraits<T>::kPairsPerVec>& r, float (&out)[VecTraits<T>::kElems]) {
    using Tr = VecTraits<T>;
#pragma unroll
    for (int h = 0; h < Tr::kPairsPerVec / 2; ++h) {
        const float4 w = *reinterpret_cast<const float4*>(s_w + e0 + 4 * h);  // permuted
        float a0, c0, a1, c1;
        Tr::pair(x, 2 * h, a0, c0);
        Tr::pair(x, 2 * h + 1, a1, c1);
        const float2 y_re = __fmul2_rn(make_float2(a0, a1), make_float2(w.x, w.y));
        const float2 y_im = __fmul2_rn(make_float2(c0, c1), make_float2(w.z, w.w));
        const float2 o_re = __ffma2_rn(y_im, r.ns[h], __fmul2_rn(y_re, r.c[h]));
        const float2 o_im = __ffma2_rn(y_im, r.c[h], __fmul2_rn(y_re, r.s[h]));
        out[4 * h] = o_re.x;
        out[4 * h + 1] = o_im.x;
        out[4 * h + 2] = o_re.y;
        out[4 * h + 3] = o_im.y;
    }
}

// The same, rounded once to the element type.
template <typename T>
__device__ __forceinline__ typename VecTraits<T>::Vec norm_rotate(
    const typename VecTraits<T>::Vec& x, const float* s_w, int e0,
    const RowRot<VecTraits<T>::kPairsPerVec>& r) {
    float out[VecTraits<T>::kElems];
    norm_rotate_f<T>(x, s_w, e0, r, out);
    return VecTraits<T>::pack_elems(out);
}

// RoPE alone (the rotation-only entry point), rounded once to the element type.
template <typename T>
__device__ __forceinline__ typename VecTraits<T>::Vec rotate_only(
    const typename VecTraits<T>::Vec& x, const float (&cs)[VecTraits<T>::kPairsPerVec],
    const float (&sn)[VecTraits<T>::kPairsPerVec]) {
    using Tr = VecTraits<T>;
    float out[Tr::kElems];
#pragma unroll
    for (int m = 0; m < Tr::kPairsPerVec; ++m) {
        float a, c;
        Tr::pair(x, m, a, c);
        out[2 * m] = a * cs[m] - c * sn[m];
        out[2 * m + 1] = a * sn[m] + c * cs[m];
    }
    return Tr::pack_elems(out);
}

// rotate_half pairing: `re_v` is a head's first-half vector at some position and
// `im_v` its second-half vector at the same position -- the real and imaginary parts of
// kElems pairs.  Both are normalised with their own weights, y = x * rs * w, and
// (y_re + i y_im) * (cos + i sin) is returned as fp32 in the two vectors' element order.
template <typename T, bool NORM>
__device__ __forceinline__ void norm_rotate_half_f(
    const typename VecTraits<T>::Vec& re_v, const typename VecTraits<T>::Vec& im_v, float rs,
    const float* s_w, int e_re, int e_im,
    const float (&cs)[VecTraits<T>::kElems], const float (&sn)[VecTraits<T>::kElems],
    float (&o_re)[VecTraits<T>::kElems], float (&o_im)[VecTraits<T>::kElems]) {
    using Tr = VecTraits<T>;
    constexpr int E = Tr::kElems;
    float wr[E], wi[E];
    if (NORM) {
#pragma unroll
        for (int c = 0; c < E / 4; ++c) {
            const float4 a = weights4(s_w, e_re + 4 * c);
            const float4 b = weights4(s_w, e_im + 4 * c);
            wr[4 * c] = a.x; wr[4 * c + 1] = a.y; wr[4 * c + 2] = a.z; wr[4 * c + 3] = a.w;
            wi[4 * c] = b.x; wi[4 * c + 1] = b.y; wi[4 * c + 2] = b.z; wi[4 * c + 3] = b.w;
        }
    }
#pragma unroll
    for (int m = 0; m < E; ++m) {
        float a = Tr::elem(re_v, m);
        float c = Tr::elem(im_v, m);
        if (NORM) {
            a = a * rs * wr[m];
            c = c * rs * wi[m];
        }
        o_re[m] = a * cs[m] - c * sn[m];
        o_im[m] = a * sn[m] + c * cs[m];
    }
}

// ---------------------------------------------------------------- FP8 E4M3 cache rows
//
// Quantize-on-append: a head's K or V row goes to the cache as E4M3 codes with one fp32
// scale.  The scale is a power of two (as in the OCP microscaling formats): the smallest
// 2^e, e >= -126, with amax / 2^e <= 448; codes are E4M3(x * 2^-e) -- an exact scaling --
// rounded to nearest even with saturation.  The lanes holding a head (at one slot) agree
// on its scale through a butterfly maximum of integer keys, two heads per shuffle; the
// head's first lane writes the scale.

// Key of a magnitude a >= 0: a's biased exponent, plus one when a's mantissa lies above
// that of 1.75 (448 = 1.75 * 2^8), so that the smallest e with a <= 448 * 2^e is
// key - 135.  The key is monotone in a, so a head's key is the maximum of its lanes'.
__device__ __forceinline__ uint32_t fp8_key(float a) {
    return (__float_as_uint(a) + 0x1FFFFFu) >> 23;
}

struct Fp8Scale {
    float scale;  // stored for the reader: x ~ value(code) * scale
    float inv;    // codes are E4M3(x * inv)
};

__device__ __forceinline__ Fp8Scale fp8_scale_from_key(uint32_t key) {
    key = max(key, 9u);  // e = key - 135 >= -126
    Fp8Scale s;
    s.scale = __uint_as_float((key - 8u) << 23);  // 2^e
    s.inv = __uint_as_float((262u - key) << 23);  // 2^-e
    return s;
}

// Three-input maximum (a single instruction on sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Scales of two heads from this lane's keys k0, k1: the keys travel packed in the halves
// of one word, reduced over groups of `lanes` lanes (a power of two <= 32).
__device__ __forceinline__ void fp8_scale_pair(uint32_t k0, uint32_t k1, int lanes,
                                               Fp8Scale& s0, Fp8Scale& s1) {
    uint32_t w = k0 | (k1 << 16);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        if (off < lanes) w = max_u16x2(w, __shfl_xor_sync(0xffffffffu, w, off));
    s0 = fp8_scale_from_key(w & 0xFFFFu);
    s1 = fp8_scale_from_key(w >> 16);
}

// Key of the largest magnitude in a vector of finite input elements (the quantizer's
// domain).  For bf16 three `max.xorsign.abs.bf16x2` reduce the four words to two
// magnitudes (the sign bits, an xor of the inputs', are masked off), compared as 16-bit
// integers; the key of a bf16 value with bits b is (b + 0x1F) >> 7, fp8_key of its fp32
// widening b << 16.
__device__ __forceinline__ uint32_t vec_key(const uint4& v) {
    uint32_t a, b, m;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(v.x), "r"(v.y));
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(b) : "r"(v.z), "r"(v.w));
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(a), "r"(b));
    m &= 0x7FFF7FFFu;
    return (max(m & 0xFFFFu, m >> 16) + 0x1Fu) >> 7;
}
__device__ __forceinline__ uint32_t vec_key(const float4& v) {
    return fp8_key(fmaxf(max3f(fabsf(v.x), fabsf(v.y), fabsf(v.z)), fabsf(v.w)));
}
// Largest magnitude of a vector of input elements (exact; for bf16 the same reduction
// as vec_key, then the larger of the two magnitudes widened to fp32).
__device__ __forceinline__ float vec_abs_max(const uint4& v) {
    uint32_t a, b, m;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(v.x), "r"(v.y));
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(b) : "r"(v.z), "r"(v.w));
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(a), "r"(b));
    m &= 0x7FFF7FFFu;
    return __uint_as_float(max(m & 0xFFFFu, m >> 16) << 16);
}
__device__ __forceinline__ float vec_abs_max(const float4& v) {
    return fmaxf(max3f(fabsf(v.x), fabsf(v.y), fabsf(v.z)), fabsf(v.w));
}

__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
    // element a in the low byte (lower address)
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

// ---------------------------------------------------------------- NVFP4 cache rows
//
// Each block of 16 consecutive elements of a head goes to the cache as 16 E2M1 codes
// (two per byte, element 2j in the low nibble) with one E4M3 block scale S, under the
// tensor's fp32 scale g: S = E4M3(amax * k) with k = 1 / (6 g), codes = E2M1(x * r) with
// r = 1 / (value(S) g) (0 when S is zero), each operation one fp32 rounding to nearest.
// r depends on S alone, so each block of threads tabulates it for the 256 codes once.
// A block of 16 elements is 2 vectors (bf16) or 4 (fp32) held by as many neighbouring
// lanes.

constexpr int kNvfp4TableFloats = 512;  // r for the 256 codes, K then V

// Value of a non-negative E4M3 code (exponent bias 7, 3 mantissa bits; field 0 is
// subnormal m * 2^-9), built from its fields.
__device__ __forceinline__ float e4m3_nonneg_value(uint32_t code) {
    const uint32_t e = (code >> 3) & 15u, m = code & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0x1p-9f;
}

__device__ __forceinline__ void fill_nvfp4_tables(const Params& p, float* s_r) {
    for (int c = threadIdx.x; c < 256; c += blockDim.x) {
        const float sv = e4m3_nonneg_value((uint32_t)c);
        s_r[c] = sv > 0.0f ? __frcp_rn(__fmul_rn(sv, p.k_global)) : 0.0f;
        s_r[256 + c] = sv > 0.0f ? __frcp_rn(__fmul_rn(sv, p.v_global)) : 0.0f;
    }
}

struct Nvfp4Scale {
    uint32_t code;  // E4M3 byte
    float r;        // 1 / (value(S) g), or 0
};

__device__ __forceinline__ Nvfp4Scale nvfp4_scale(float amax, float inv6g, const float* s_r) {
    Nvfp4Scale s;
    s.code = e4m3x2(__fmul_rn(amax, inv6g), 0.0f) & 0xFFu;
    s.r = s_r[s.code];
    return s;
}

// E2M1 codes of 8 values in one 32-bit word, element 0 in the low nibble.
__device__ __forceinline__ uint32_t e2m1x8(float2 a, float2 b, float2 c, float2 d) {
    uint32_t r;
    asm("{\n .reg .b8 b0, b1, b2, b3;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
        " mov.b32 %0, {b0, b1, b2, b3};\n}"
        : "=r"(r)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y), "f"(d.x), "f"(d.y));
    return r;
}

// Store the codes of one vector at vector index vi of an NVFP4 cache (E/2 bytes per vector).
__device__ __forceinline__ void store_fp4(void* cache, int64_t vi, const float (&v)[8], float r) {
    const float2 r2 = make_float2(r, r);
    const uint32_t c = e2m1x8(__fmul2_rn(make_float2(v[0], v[1]), r2),
                              __fmul2_rn(make_float2(v[2], v[3]), r2),
                              __fmul2_rn(make_float2(v[4], v[5]), r2),
                              __fmul2_rn(make_float2(v[6], v[7]), r2));
    __stcs(reinterpret_cast<unsigned int*>(cache) + vi, c);
}
__device__ __forceinline__ void store_fp4(void* cache, int64_t vi, const float (&v)[4], float r) {
    const float2 r2 = make_float2(r, r);
    const float2 z = make_float2(0.0f, 0.0f);
    const uint32_t c = e2m1x8(__fmul2_rn(make_float2(v[0], v[1]), r2),
                              __fmul2_rn(make_float2(v[2], v[3]), r2), z, z);
    __stcs(reinterpret_cast<unsigned short*>(cache) + vi, (unsigned short)c);
}

// Maximum over the `lanes` neighbouring lanes that hold one block (1, 2 or 4).
__device__ __forceinline__ float block_max(float x, int lanes) {
    for (int off = 1; off < lanes; off <<= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
    return x;
}

// Store E codes of one vector at vector index vi of an FP8 cache (E bytes per vector);
// the values are scaled two at a time (packed fp32x2 multiplies).
// E4M3 codes of four values in one 32-bit word, a in the low byte: two conversions into
// the halves of one register.
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
    uint32_t r;
    asm("{\n"
        "  .reg .b16 lo, hi;\n"
        "  cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n"
        "  cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n"
        "  mov.b32 %0, {lo, hi};\n"
        "}"
        : "=r"(r)
        : "f"(a), "f"(b), "f"(c), "f"(d));
    return r;
}
__device__ __forceinline__ uint32_t e4m3x4_scaled(float a, float b, float c, float d,
                                                  float2 inv2) {
    const float2 x = __fmul2_rn(make_float2(a, b), inv2);
    const float2 y = __fmul2_rn(make_float2(c, d), inv2);
    return e4m3x4(x.x, x.y, y.x, y.y);
}
__device__ __forceinline__ void store_fp8(void* cache, int64_t vi, const float (&v)[8],
                                          float inv) {
    const float2 inv2 = make_float2(inv, inv);
    uint2 c;
    c.x = e4m3x4_scaled(v[0], v[1], v[2], v[3], inv2);
    c.y = e4m3x4_scaled(v[4], v[5], v[6], v[7], inv2);
    __stcs(reinterpret_cast<uint2*>(cache) + vi, c);
}
__device__ __forceinline__ void store_fp8(void* cache, int64_t vi, const float (&v)[4],
                                          float inv) {
    const uint32_t c = e4m3x4_scaled(v[0], v[1], v[2], v[3], make_float2(inv, inv));
    __stcs(reinterpret_cast<unsigned int*>(cache) + vi, c);
}

template <int E>
__device__ __forceinline__ float abs_max(const float (&v)[E]) {
    static_assert(E == 4 || E == 8, "vectors hold 4 or 8 elements");
    float m = max3f(fabsf(v[0]), fabsf(v[1]), fabsf(v[2]));
    if constexpr (E == 4) return fmaxf(m, fabsf(v[3]));
    m = max3f(m, fabsf(v[3]), fabsf(v[4]));
    m = max3f(m, fabsf(v[5]), fabsf(v[6]));
    return fmaxf(m, fabsf(v[7]));
}

__device__ __forceinline__ void stage_weights(const Params& p, float* s_wq, float* s_wk) {
    // dim is a multiple of 128, so float4 copies cover it
    const float4* gq = reinterpret_cast<const float4*>(p.q_w);
    const float4* gk = reinterpret_cast<const float4*>(p.k_w);
    float4* sq4 = reinterpret_cast<float4*>(s_wq);
    float4* sk4 = reinterpret_cast<float4*>(s_wk);
    for (int e = threadIdx.x; e < p.dim / 4; e += blockDim.x) {
        const float4 a = __ldg(gq + e), b = __ldg(gk + e);
        sq4[e] = make_float4(a.x, a.z, a.y, a.w);  // (w0, w2, w1, w3): see weights4
        sk4[e] = make_float4(b.x, b.z, b.y, b.w);
    }
}

// ---------------------------------------------------------------- per-row output

// The two bf16 halves of u (low half first) times a power of two s (given as its bf16
// bits), as fp32: one mixed-precision FMA per element widens and scales at once.  The
// product of a bf16 value and a power of two is exact in fp32 (the -0 addend keeps the
// sign of a zero product), so this equals widening and then multiplying in fp32.
__device__ __forceinline__ float2 bf16x2_times_pow2(uint32_t u, unsigned short s) {
    float2 r;
    asm("{\n"
        "  .reg .b16 lo, hi;\n"
        "  mov.b32 {lo, hi}, %2;\n"
        "  fma.rn.f32.bf16 %0, lo, %3, 0f80000000;\n"
        "  fma.rn.f32.bf16 %1, hi, %3, 0f80000000;\n"
        "}"
        : "=f"(r.x), "=f"(r.y)
        : "r"(u), "h"(s));
    return r;
}

// Quantize one vector of V (its input elements) to the FP8 cache.
template <typename T>
__device__ __forceinline__ void store_v_fp8(void* vc, int64_t vi,
                                            const typename VecTraits<T>::Vec& x, float inv) {
    using Tr = VecTraits<T>;
    if constexpr (Tr::kElems == 8) {
        // bf16: inv is a power of two, so its bf16 bits are the top half of its fp32 bits
        const unsigned short s = (unsigned short)(__float_as_uint(inv) >> 16);
        const float2 a = bf16x2_times_pow2(x.x, s), b = bf16x2_times_pow2(x.y, s);
        const float2 c = bf16x2_times_pow2(x.z, s), d = bf16x2_times_pow2(x.w, s);
        uint2 w;
        w.x = e4m3x4(a.x, a.y, b.x, b.y);
        w.y = e4m3x4(c.x, c.y, d.x, d.y);
        __stcs(reinterpret_cast<uint2*>(vc) + vi, w);
    } else {
        float v[Tr::kElems];
#pragma unroll
        for (int e = 0; e < Tr::kElems; ++e) v[e] = Tr::elem(x, e);
        store_fp8(vc, vi, v, inv);
    }
}

// Normalise, rotate and store this thread's vectors of one row: q_out, and in the fused
// mode the K row into the cache.  With rotate_half pairing slots 2m and 2m+1 hold the two
// halves of the same pairs (see slot_vec).  V goes to a same-dtype cache through
// store_v_row; with an FP8 or NVFP4 cache (CF) it is quantized here, beside K: the K values stay
// fp32 until they are quantized, and the K and V keys of one head travel in one shuffle
// word.  Every lane of the warp takes part in the head-wise maximum, whether its slots
// hold vectors or not.
template <typename T, int VPT, int PAIR, int MODE, int CF>
__device__ __forceinline__ void emit_row(
    const Params& p, int t, const RowPos& pos, int64_t row_vec,
    const typename VecTraits<T>::Vec (&xq)[VPT], const typename VecTraits<T>::Vec (&xk)[VPT],
    const typename VecTraits<T>::Vec (&xv)[VPT],
    float rq, float rk, const float* s_wq, const float* s_wk,
    const float (&cs)[PairCount<T, PAIR>::value], const float (&sn)[PairCount<T, PAIR>::value],
    typename VecTraits<T>::Vec* qo, typename VecTraits<T>::Vec* kc,
    typename VecTraits<T>::Vec* vc, const float* s_r = nullptr) {
    using Tr = VecTraits<T>;
    constexpr int EPV = Tr::kElems;
    constexpr bool NORM = MODE == kModeFused;
    constexpr bool QUANT = MODE == kModeFused && CF == kCacheFp8;
    constexpr bool QUANT4 = MODE == kModeFused && CF == kCacheNvfp4;
    constexpr int VPH = Tr::kVecsPerHead;
    constexpr int VPB = 16 / EPV;  // vectors (lanes) per NVFP4 block
    if constexpr (PAIR == kPairAdjacent) {
        // q first, for every slot, then K (and V where it is quantized): one row rotation
        // (RowRot) is live at a time
        if constexpr (NORM) {
            const RowRot<Tr::kPairsPerVec> rot_q = row_rot(rq, cs, sn);
#pragma unroll
            for (int s = 0; s < VPT; ++s) {
                const int idx = slot_vec<T, PAIR>(t, s, p.tpr);
                if (idx < p.dim_vecs && (!kDeviceChecks || pos.ok))
                    store_out(qo + row_vec + idx, norm_rotate<T>(xq[s], s_wq, idx * EPV, rot_q));
            }
        } else {
#pragma unroll
            for (int s = 0; s < VPT; ++s) {
                const int idx = slot_vec<T, PAIR>(t, s, p.tpr);
                if (idx < p.dim_vecs && (!kDeviceChecks || pos.ok))
                    store_out(qo + row_vec + idx, rotate_only<T>(xq[s], cs, sn));
            }
        }
        if constexpr (MODE == kModeFused) {
            const RowRot<Tr::kPairsPerVec> rot_k = row_rot(rk, cs, sn);
#pragma unroll
            for (int s = 0; s < VPT; ++s) {
                const int idx = slot_vec<T, PAIR>(t, s, p.tpr);
                const bool valid = idx < p.dim_vecs && (!kDeviceChecks || pos.ok);
                const int e0 = idx * EPV;
                if constexpr (QUANT && VPT <= 3) {
                    // slots s and s + 1 at once: two key words, two interleaved butterflies
                    // (measured on B200: 3% faster at three vectors per thread; slower at
                    // four, where the extra live values cost more than the overlap gains)
                    if (s % 2 == 0) {
                        constexpr int kPair = 2;
                        float o[kPair][EPV];
                        uint32_t wkey[kPair] = {0u, 0u};
                        int id[kPair];
                        bool ok[kPair];
#pragma unroll
                        for (int j = 0; j < kPair; ++j) {
                            const int sj = s + j < VPT ? s + j : s;
                            id[j] = slot_vec<T, PAIR>(t, s + j, p.tpr);
                            ok[j] = s + j < VPT && id[j] < p.dim_vecs &&
                                    (!kDeviceChecks || pos.ok);
                            if (ok[j]) {
                                norm_rotate_f<T>(xk[sj], s_wk, id[j] * EPV, rot_k, o[j]);
                                wkey[j] = fp8_key(abs_max<EPV>(o[j])) | (vec_key(xv[sj]) << 16);
                            }
                        }
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1)
                            if (off < VPH) {
#pragma unroll
                                for (int j = 0; j < kPair; ++j)
                                    wkey[j] = max_u16x2(
                                        wkey[j], __shfl_xor_sync(0xffffffffu, wkey[j], off));
                            }
#pragma unroll
                        for (int j = 0; j < kPair; ++j) {
                            if (!ok[j]) continue;
                            const int sj = s + j < VPT ? s + j : s;
                            const Fp8Scale sk = fp8_scale_from_key(wkey[j] & 0xFFFFu);
                            const Fp8Scale sv = fp8_scale_from_key(wkey[j] >> 16);
                            const int64_t vi = cache_vec_index(p, pos, id[j]);
                            store_fp8(kc, vi, o[j], sk.inv);
                            store_v_fp8<T>(vc, vi, xv[sj], sv.inv);
                            if ((id[j] & (VPH - 1)) == 0) {
                                const int64_t si = cache_scale_index(p, pos, id[j] / VPH);
                                __stcs(p.k_scale + si, sk.scale);
                                __stcs(p.v_scale + si, sv.scale);
                            }
                        }
                    }
                } else if constexpr (QUANT) {
                    float o[EPV];
                    uint32_t kk = 0, kv = 0;
                    if (valid) {
                        norm_rotate_f<T>(xk[s], s_wk, e0, rot_k, o);
                        kk = fp8_key(abs_max<EPV>(o));
                        kv = vec_key(xv[s]);
                    }
                    Fp8Scale sk, sv;
                    fp8_scale_pair(kk, kv, VPH, sk, sv);
                    if (valid) {
                        const int64_t vi = cache_vec_index(p, pos, idx);
                        store_fp8(kc, vi, o, sk.inv);
                        store_v_fp8<T>(vc, vi, xv[s], sv.inv);
                        if ((idx & (VPH - 1)) == 0) {
                            const int64_t si = cache_scale_index(p, pos, idx / VPH);
                            __stcs(p.k_scale + si, sk.scale);
                            __stcs(p.v_scale + si, sv.scale);
                        }
                    }
                } else if constexpr (QUANT4) {
                    float o[EPV];
                    float ak = 0.0f, av = 0.0f;
                    if (valid) {
                        norm_rotate_f<T>(xk[s], s_wk, e0, rot_k, o);
                        ak = abs_max<EPV>(o);
                        av = vec_abs_max(xv[s]);
                    }
                    ak = block_max(ak, VPB);
                    av = block_max(av, VPB);
                    if (valid) {
                        const Nvfp4Scale sk = nvfp4_scale(ak, p.k_inv6g, s_r);
                        const Nvfp4Scale sv = nvfp4_scale(av, p.v_inv6g, s_r + 256);
                        const int64_t vi = cache_vec_index(p, pos, idx);
                        float v[EPV];
#pragma unroll
                        for (int e = 0; e < EPV; ++e) v[e] = Tr::elem(xv[s], e);
                        store_fp4(kc, vi, o, sk.r);
                        store_fp4(vc, vi, v, sv.r);
                        if ((idx & (VPB - 1)) == 0) {
                            __stcs(reinterpret_cast<char*>(p.k_bscale + vi / VPB), (char)sk.code);
                            __stcs(reinterpret_cast<char*>(p.v_bscale + vi / VPB), (char)sv.code);
                        }
                    }
                } else if (valid) {
                    store_out(kc + cache_vec_index(p, pos, idx),
                              norm_rotate<T>(xk[s], s_wk, e0, rot_k));
                }
            }
        }
    } else {
        static_assert(VPT % 2 == 0, "rotate_half slots come in twos");
#pragma unroll
        for (int s = 0; s < VPT; s += 2) {
            const int i_re = slot_vec<T, PAIR>(t, s, p.tpr);
            const int i_im = slot_vec<T, PAIR>(t, s + 1, p.tpr);
            const bool valid = i_re < p.dim_vecs && (!kDeviceChecks || pos.ok);
            float o_re[EPV], o_im[EPV];
            if (valid) {
                norm_rotate_half_f<T, NORM>(xq[s], xq[s + 1], rq, s_wq, i_re * EPV, i_im * EPV,
                                            cs, sn, o_re, o_im);
                store_out(qo + row_vec + i_re, Tr::pack_elems(o_re));
                store_out(qo + row_vec + i_im, Tr::pack_elems(o_im));
            }
            if constexpr (MODE == kModeFused) {
                if (valid)
                    norm_rotate_half_f<T, true>(xk[s], xk[s + 1], rk, s_wk, i_re * EPV,
                                                i_im * EPV, cs, sn, o_re, o_im);
                if constexpr (QUANT4) {
                    // i_re and i_im lie in different blocks: each reduces over its own lanes
                    float a_re = 0.0f, a_im = 0.0f, v_re = 0.0f, v_im = 0.0f;
                    if (valid) {
                        a_re = abs_max<EPV>(o_re);
                        a_im = abs_max<EPV>(o_im);
                        v_re = vec_abs_max(xv[s]);
                        v_im = vec_abs_max(xv[s + 1]);
                    }
                    a_re = block_max(a_re, VPB);
                    a_im = block_max(a_im, VPB);
                    v_re = block_max(v_re, VPB);
                    v_im = block_max(v_im, VPB);
                    if (valid) {
                        const int64_t vr = cache_vec_index(p, pos, i_re);
                        const int64_t vm = cache_vec_index(p, pos, i_im);
                        const Nvfp4Scale k_re = nvfp4_scale(a_re, p.k_inv6g, s_r);
                        const Nvfp4Scale k_im = nvfp4_scale(a_im, p.k_inv6g, s_r);
                        const Nvfp4Scale s_re = nvfp4_scale(v_re, p.v_inv6g, s_r + 256);
                        const Nvfp4Scale s_im = nvfp4_scale(v_im, p.v_inv6g, s_r + 256);
                        float v[EPV];
                        store_fp4(kc, vr, o_re, k_re.r);
                        store_fp4(kc, vm, o_im, k_im.r);
#pragma unroll
                        for (int e = 0; e < EPV; ++e) v[e] = Tr::elem(xv[s], e);
                        store_fp4(vc, vr, v, s_re.r);
#pragma unroll
                        for (int e = 0; e < EPV; ++e) v[e] = Tr::elem(xv[s + 1], e);
                        store_fp4(vc, vm, v, s_im.r);
                        if ((i_re & (VPB - 1)) == 0) {
                            __stcs(reinterpret_cast<char*>(p.k_bscale + vr / VPB), (char)k_re.code);
                            __stcs(reinterpret_cast<char*>(p.k_bscale + vm / VPB), (char)k_im.code);
                            __stcs(reinterpret_cast<char*>(p.v_bscale + vr / VPB), (char)s_re.code);
                            __stcs(reinterpret_cast<char*>(p.v_bscale + vm / VPB), (char)s_im.code);
                        }
                    }
                } else if constexpr (QUANT) {
                    uint32_t kk = 0, kv = 0;
                    if (valid) {
                        kk = fp8_key(fmaxf(abs_max<EPV>(o_re), abs_max<EPV>(o_im)));
                        kv = max(vec_key(xv[s]), vec_key(xv[s + 1]));
                    }
                    Fp8Scale sk, sv;
                    fp8_scale_pair(kk, kv, VPH / 2, sk, sv);
                    if (valid) {
                        const int64_t vr = cache_vec_index(p, pos, i_re);
                        const int64_t vm = cache_vec_index(p, pos, i_im);
                        store_fp8(kc, vr, o_re, sk.inv);
                        store_fp8(kc, vm, o_im, sk.inv);
                        store_v_fp8<T>(vc, vr, xv[s], sv.inv);
                        store_v_fp8<T>(vc, vm, xv[s + 1], sv.inv);
                        if ((i_re & (VPH - 1)) == 0) {
                            const int64_t si = cache_scale_index(p, pos, i_re / VPH);
                            __stcs(p.k_scale + si, sk.scale);
                            __stcs(p.v_scale + si, sv.scale);
                        }
                    }
                } else if (valid) {
                    store_out(kc + cache_vec_index(p, pos, i_re), Tr::pack_elems(o_re));
                    store_out(kc + cache_vec_index(p, pos, i_im), Tr::pack_elems(o_im));
                }
            }
        }
    }
}

// Store this thread's vectors of one row of V to a same-dtype cache: a bit copy.
template <typename T, int VPT, int PAIR>
__device__ __forceinline__ void store_v_row(const Params& p, int t, const RowPos& pos,
                                            const typename VecTraits<T>::Vec (&xv)[VPT],
                                            typename VecTraits<T>::Vec* vc) {
#pragma unroll
    for (int s = 0; s < VPT; ++s) {
        const int idx = slot_vec<T, PAIR>(t, s, p.tpr);
        if (idx < p.dim_vecs && (!kDeviceChecks || pos.ok))
            store_out(vc + cache_vec_index(p, pos, idx), xv[s]);
    }
}

// ---------------------------------------------------------------- head-scatter stores
//
// The sequence-parallel all-to-all (sequence gather, head scatter) folded into the step:
// a rank holds all heads of its token slice, and each head's q, K and V go straight to
// the rank that owns the head -- q to row (i - sp_q_row0) of that rank's q buffer, K and
// V to its caches at the token's cache row -- as plain stores (through peer mappings when
// the destination is another GPU).  The destination of a slot depends on the thread
// only: code = (rank << 16) | vector index within the destination's token row.

__device__ __forceinline__ int sp_code(const Params& p, int idx) {
    const int vph = 1 << p.vph_log2;
    const int d = (idx >> p.vph_log2) / p.sp_heads;
    return (d << 16) | (idx - d * p.sp_heads * vph);
}

// Vector index of local vector dv of a cache row in a destination cache of sp_heads heads.
__device__ __forceinline__ int64_t sp_cache_index(const Params& p, const RowPos& pos, int dv) {
    if (!p.cache_head_major)
        return ((pos.b * p.cache_tokens + pos.crow) * p.sp_heads << p.vph_log2) + dv;
    const int nl = dv >> p.vph_log2;
    const int v = dv & ((1 << p.vph_log2) - 1);
    return (((pos.b * p.sp_heads + nl) * p.cache_tokens + pos.crow) << p.vph_log2) + v;
}

template <typename T, int VPT>
__device__ __forceinline__ void store_v_row_sp(const Params& p, int t, const RowPos& pos,
                                               const typename VecTraits<T>::Vec (&xv)[VPT],
                                               const int (&dst)[VPT], void* const* s_sp) {
    using Vec = typename VecTraits<T>::Vec;
#pragma unroll
    for (int s = 0; s < VPT; ++s) {
        if (slot_vec<T, kPairAdjacent>(t, s, p.tpr) < p.dim_vecs && (!kDeviceChecks || pos.ok)) {
            Vec* vd = reinterpret_cast<Vec*>(s_sp[3 * (dst[s] >> 16) + 2]);
            store_out(vd + sp_cache_index(p, pos, dst[s] & 0xFFFF), xv[s]);
        }
    }
}

template <typename T, int VPT>
__device__ __forceinline__ void emit_row_sp(
    const Params& p, int t, const RowPos& pos,
    const typename VecTraits<T>::Vec (&xq)[VPT], const typename VecTraits<T>::Vec (&xk)[VPT],
    float rq, float rk, const float* s_wq, const float* s_wk,
    const float (&cs)[PairCount<T, kPairAdjacent>::value],
    const float (&sn)[PairCount<T, kPairAdjacent>::value], const int (&dst)[VPT],
    void* const* s_sp) {
    using Tr = VecTraits<T>;
    using Vec = typename Tr::Vec;
    const int64_t q_row = (pos.b * p.sp_q_rows + (pos.i - p.sp_q_row0)) * p.sp_heads
                          << p.vph_log2;
    bool ok = true;
    if constexpr (kDeviceChecks) {
        ok = pos.ok && pos.i >= p.sp_q_row0 && pos.i - p.sp_q_row0 < p.sp_q_rows;
        if (pos.ok && !ok) record_index_error(p);
    }
    const RowRot<Tr::kPairsPerVec> rot_q = row_rot(rq, cs, sn);
#pragma unroll
    for (int s = 0; s < VPT; ++s) {
        const int idx = slot_vec<T, kPairAdjacent>(t, s, p.tpr);
        if (idx < p.dim_vecs && ok) {
            Vec* qd = reinterpret_cast<Vec*>(s_sp[3 * (dst[s] >> 16)]);
            store_out(qd + q_row + (dst[s] & 0xFFFF),
                      norm_rotate<T>(xq[s], s_wq, idx * Tr::kElems, rot_q));
        }
    }
    const RowRot<Tr::kPairsPerVec> rot_k = row_rot(rk, cs, sn);
#pragma unroll
    for (int s = 0; s < VPT; ++s) {
        const int idx = slot_vec<T, kPairAdjacent>(t, s, p.tpr);
        if (idx < p.dim_vecs && ok) {
            Vec* kd = reinterpret_cast<Vec*>(s_sp[3 * (dst[s] >> 16) + 1]);
            store_out(kd + sp_cache_index(p, pos, dst[s] & 0xFFFF),
                      norm_rotate<T>(xk[s], s_wk, idx * Tr::kElems, rot_k));
        }
    }
}

// ---------------------------------------------------------------- register kernel

// This thread's vectors of one tensor's token row u.
template <typename T, int VPT, int PAIR>
__device__ __forceinline__ void load_vecs(const Params& p, int t, int64_t u,
                                          const typename VecTraits<T>::Vec* g,
                                          typename VecTraits<T>::Vec (&x)[VPT]) {
    const int64_t row_vec = u * p.dim_vecs;
#pragma unroll
    for (int s = 0; s < VPT; ++s) {
        const int idx = slot_vec<T, PAIR>(t, s, p.tpr);
        if (idx < p.dim_vecs) x[s] = load_stream(g + row_vec + idx);
    }
}

template <typename T, int VPT, int TRIG, int MODE, int PAIR, int CF>
__global__ void __launch_bounds__(VPT > 4 ? kMaxBlockThreads / 2 : kMaxBlockThreads)
qk_norm_rope_kernel(const Params p) {
    using Tr = VecTraits<T>;
    using Vec = typename Tr::Vec;
    constexpr int NP = PairCount<T, PAIR>::value;
    constexpr bool FUSED = MODE != kModeApply;
    constexpr bool SP = MODE == kModeFusedSP;
    constexpr bool HAS_V = FUSED && MODE != kModeFusedNoV;
    constexpr int EMIT_MODE = MODE == kModeFusedNoV ? kModeFused : MODE;
    static_assert(HAS_V || !FUSED || CF == kCacheSame, "no-V step: same-dtype K cache");
    static_assert(!SP || (PAIR == kPairAdjacent && CF == kCacheSame),
                  "head-scatter stores: adjacent pairing, same-dtype caches");

    // dynamic shared memory: [SP: destination table | NVFP4: reciprocal tables]
    // [q, k norm weights] [team partials]
    constexpr bool FP4 = CF == kCacheNvfp4;
    extern __shared__ float4 smem4[];
    void** s_sp = reinterpret_cast<void**>(smem4);
    float* s_r = reinterpret_cast<float*>(smem4);
    float* s_wq = reinterpret_cast<float*>(
        smem4 + (SP ? 3 * kMaxRanks / 2 : FP4 ? kNvfp4TableFloats / 4 : 0));
    float* s_wk = s_wq + (FUSED ? p.dim : 0);
    float2* s_part = reinterpret_cast<float2*>(s_wk + (FUSED ? p.dim : 0));

    const int tid = threadIdx.x;
    const int team = tid / p.tpr;
    const int t = tid - team * p.tpr;
    const int lane = tid & 31;
    const int warp_in_team = t >> 5;
    const int warps_per_team = p.tpr >> 5;

    const Vec* qg = reinterpret_cast<const Vec*>(p.q);
    const Vec* kg = reinterpret_cast<const Vec*>(p.k);
    const Vec* vg = reinterpret_cast<const Vec*>(p.v);
    Vec* qo = reinterpret_cast<Vec*>(p.q_out);
    Vec* kc = reinterpret_cast<Vec*>(p.k_cache);
    Vec* vc = reinterpret_cast<Vec*>(p.v_cache);
    const int64_t stride = (int64_t)gridDim.x * p.teams;
    const int64_t u0 = (int64_t)blockIdx.x * p.teams + team;

    pdl_launch_dependents();
    pdl_wait_previous_grid();
    // The team's first row is requested before the block stages its weights, so the two
    // latencies overlap instead of adding up at the start of every launch.
    Vec xq[VPT], xk[VPT], xv[VPT];
    if (u0 < p.units) {
        load_vecs<T, VPT, PAIR>(p, t, u0, qg, xq);
        if (FUSED) load_vecs<T, VPT, PAIR>(p, t, u0, kg, xk);
        if (HAS_V) load_vecs<T, VPT, PAIR>(p, t, u0, vg, xv);
    }
    if (FUSED) {
        if constexpr (SP) {
#pragma unroll
            for (int j = 0; j < 3 * kMaxRanks; ++j)
                if (tid == j) s_sp[j] = p.sp_dst[j];  // constant indices into the parameters
        }
        if constexpr (FP4) fill_nvfp4_tables(p, s_r);
        stage_weights(p, s_wq, s_wk);
        __syncthreads();
    }
    const PairCols<NP> pi = pair_cols<NP>(p, first_pair<T, PAIR>(t % Tr::kVecsPerHead));
    int dst[VPT];
    if constexpr (SP) {
#pragma unroll
        for (int s = 0; s < VPT; ++s) dst[s] = sp_code(p, slot_vec<T, PAIR>(t, s, p.tpr));
    }

    int parity = 0;
    for (int64_t u = u0; u < p.units; u += stride) {
        const RowPos pos = decode_row(p, u);
        const int64_t row_vec = u * p.dim_vecs;
        float cs[NP], sn[NP];
        pair_trig<TRIG>(p, pi, pos, cs, sn);

        float rq = 1.0f, rk = 1.0f;
        if (FUSED) {
            if constexpr (SP) store_v_row_sp<T, VPT>(p, t, pos, xv, dst, s_sp);
            else if constexpr (CF == kCacheSame && HAS_V)
                store_v_row<T, VPT, PAIR>(p, t, pos, xv, vc);
            float sq, sk;
            partial_sum_squares<T, VPT, PAIR>(xq, xk, t, p.tpr, p.dim_vecs, sq, sk);
            const float2 tot = team_sum(sq, sk, s_part, team, p.teams, warp_in_team,
                                        warps_per_team, lane, p.tpr, parity);
            rq = rsqrtf(fmaf(tot.x, p.inv_dim, p.eps));
            rk = rsqrtf(fmaf(tot.y, p.inv_dim, p.eps));
        }
        if constexpr (SP)
            emit_row_sp<T, VPT>(p, t, pos, xq, xk, rq, rk, s_wq, s_wk, cs, sn, dst, s_sp);
        else
            emit_row<T, VPT, PAIR, EMIT_MODE, CF>(p, t, pos, row_vec, xq, xk, xv, rq, rk,
                                                  s_wq, s_wk, cs, sn, qo, kc, vc, s_r);
        // The team's next row, requested after this row's stores: one row in registers at a
        // time keeps the blocks per SM up.  Measured on B200: a second row prefetched into
        // registers cost 20-40% (lost occupancy), and refilling each tensor's registers as
        // soon as the row was done with them cost 8-15% (480P and 720P chunks).
        if (u + stride < p.units) {
            load_vecs<T, VPT, PAIR>(p, t, u + stride, qg, xq);
            if (FUSED) load_vecs<T, VPT, PAIR>(p, t, u + stride, kg, xk);
            if (HAS_V) load_vecs<T, VPT, PAIR>(p, t, u + stride, vg, xv);
        }
    }
}

// ---------------------------------------------------------------- output all-to-all
//
// The exchange after attention (Algorithm 3, last step): this rank's o [B][L][hl][D] --
// every token for its own heads -- goes out token by token to the rank whose slice holds
// the token, at head offset rank * hl of that rank's [B][slice][N][D] buffer.  A bit copy
// in W-byte units (16, or 32 when every pointer allows it); the source and each
// destination row segment are contiguous, so loads and stores are coalesced on both
// sides.  Each thread takes U units a step, all U loads issued before the first store,
// so that U units per thread are in flight.

struct SpOutParams {
    const unsigned char* o;
    unsigned char* out[kMaxRanks];
    int64_t cuts[kMaxRanks + 1];
    int64_t L;
    int64_t total;        // B * L * row_units
    int ranks;
    int rank;
    int row_units;        // units of one token of o (hl heads)
    int out_row_units;    // units of one token of an output (all heads)
    int small;            // total < 2^31: 32-bit index arithmetic
    FastDiv div_row, div_L;
};

template <int W>
struct CopyUnit;
template <>
struct CopyUnit<16> {
    uint4 v;
    __device__ __forceinline__ void load(const unsigned char* p) {
        v = __ldcs(reinterpret_cast<const uint4*>(p));
    }
    __device__ __forceinline__ void store(unsigned char* p) const {
        __stcs(reinterpret_cast<uint4*>(p), v);
    }
};
template <>
struct CopyUnit<32> {  // one 256-bit access (sm_100)
    uint32_t w[8];
    __device__ __forceinline__ void load(const unsigned char* p) {
        asm volatile("ld.global.cs.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]),
                       "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                     : "l"(p));
    }
    __device__ __forceinline__ void store(unsigned char* p) const {
        asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                     ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]),
                       "r"(w[5]), "r"(w[6]), "r"(w[7])
                     : "memory");
    }
};

template <int W, int U>
__global__ void sp_output_all_to_all_kernel(const SpOutParams p) {
    pdl_launch_dependents();
    pdl_wait_previous_grid();
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    for (int64_t v0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v0 < p.total;
         v0 += U * step) {
        CopyUnit<W> x[U];
#pragma unroll
        for (int j = 0; j < U; ++j)
            if (v0 + j * step < p.total) x[j].load(p.o + (v0 + j * step) * W);
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int64_t v = v0 + j * step;
            if (v >= p.total) break;
            int64_t row, b, i;
            if (p.small) {
                const uint32_t r32 = fast_div((uint32_t)v, p.div_row);
                const uint32_t b32 = fast_div(r32, p.div_L);
                row = r32;
                b = b32;
                i = r32 - b32 * (uint32_t)p.L;
            } else {
                row = v / p.row_units;
                b = row / p.L;
                i = row - b * p.L;
            }
            const int c = (int)(v - row * p.row_units);
            int d = 0;
#pragma unroll
            for (int r = 0; r < kMaxRanks; ++r)
                if (r < p.ranks && i >= p.cuts[r] && i < p.cuts[r + 1]) d = r;
            const int64_t rows_d = p.cuts[d + 1] - p.cuts[d];
            const int64_t dst = ((b * rows_d + (i - p.cuts[d])) * p.out_row_units) +
                                (int64_t)p.rank * p.row_units + c;
            x[j].store(p.out[d] + dst * W);
        }
    }
}

// One thread per index: (t_g, h, w, cache row) as int64.
__global__ void decode_positions_kernel(int64_t token_begin, int64_t n_tok, int64_t frame_offset,
                                        int64_t hw, int W, int H, int64_t cache_tokens,
                                        int64_t slot, int64_t* out) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= n_tok) return;
    const int64_t i = token_begin + r;
    const int64_t t_local = i / hw;
    const int64_t rem = i - t_local * hw;
    const int64_t h = rem / W;
    const int64_t w = rem - h * W;
    (void)H;
    out[4 * r + 0] = frame_offset + t_local;
    out[4 * r + 1] = h;
    out[4 * r + 2] = w;
    out[4 * r + 3] = (slot + i) % cache_tokens;
}

}  // namespace rope3d
