// rope3d_kernels.cuh -- sm_100a kernels of the fused QK-RMSNorm + causal 3D RoPE +
// KV-cache append step ("Accelerating Video Generation Inference with Sequential-
// Parallel 3D Positional Encoding Using a Global Time Index", Yuan & Li: Sections
// 3.3.1-3.3.3, Algorithm 2, Algorithm 3 steps 3 and 5).
//
// The step moves 6 * N * 128 elements per token and does ~15 flops per element of
// q and k, so it is bound by HBM bandwidth, not by arithmetic: no tensor cores.
// Design:
//   * A "team" of TPR threads (a multiple of 32) owns one token row at a time.
//     Thread t of a team holds the 16-byte vectors t, t + TPR, t + 2 TPR, ... of the
//     row (coalesced 128-bit accesses).  TPR is a multiple of the vectors per head,
//     so a thread always sees the same position inside a head, hence the same few
//     complex pairs: its cos/sin are computed once per row and reused for every head
//     it holds and for both q and k.
//   * RMSNorm needs the sum of squares of the whole N*128 row before any output, so
//     a thread keeps its vectors of q, k and v in registers; the sum is a fixed
//     warp butterfly followed, for multi-warp teams, by a fixed-order sum of the
//     warps' partials (one named barrier per row, double-buffered partials).  The
//     reduction order depends only on N and the dtype, never on the token range or
//     the grid, so any slice of a sequence is bit-identical to the whole.
//   * Blocks are persistent (grid = SMs x resident blocks); each block stages the
//     two RMSNorm weight vectors in shared memory once and its teams stride over
//     the (batch, token) rows.  Inputs are read with evict-first loads; the V row is
//     stored as soon as it arrives, K and Q once normalised and rotated.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rope3d {

constexpr int kHeadDim = 128;
constexpr int kPairs = kHeadDim / 2;
constexpr int kMaxTeamsPerBlock = 15;  // named barriers 1..15 (0 is __syncthreads)
constexpr int kMaxBlockThreads = 512;  // leaves up to 128 registers per thread

enum Mode : int { kModeFused = 0, kModeApply = 1 };
enum Trig : int { kTrigTable = 0, kTrigOnTheFly = 1 };

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
    int64_t n_tok;        // rows per batch sample
    int64_t units;        // B * n_tok rows in total
    int64_t token_begin;
    int64_t frame_offset;
    int64_t cache_tokens;
    int64_t slot;
    int64_t hw;           // H * W
    int H;
    int W;
    int dim;              // N * 128 elements per row
    int dim_vecs;         // 16-byte vectors per row
    int tpr;              // threads per team (multiple of 32)
    int teams;            // teams per block
    float eps;
    float inv_dim;        // 1 / dim
    int n_t, n_h, n_w;
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
};

// ---------------------------------------------------------------- memory helpers

__device__ __forceinline__ uint4 load_stream(const uint4* p) { return __ldcs(p); }
__device__ __forceinline__ float4 load_stream(const float4* p) { return __ldcs(p); }
__device__ __forceinline__ void store_out(uint4* p, const uint4& v) { *p = v; }
__device__ __forceinline__ void store_out(float4* p, const float4& v) { *p = v; }

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

// ---------------------------------------------------------------- the kernel

template <typename T, int VPT, int TRIG, int MODE>
__global__ void __launch_bounds__(kMaxBlockThreads)
qk_norm_rope_kernel(const Params p) {
    using Tr = VecTraits<T>;
    using Vec = typename Tr::Vec;
    constexpr int PPV = Tr::kPairsPerVec;
    constexpr int EPV = 2 * PPV;  // elements per vector

    extern __shared__ float4 smem4[];
    float* s_wq = reinterpret_cast<float*>(smem4);
    float* s_wk = s_wq + (MODE == kModeFused ? p.dim : 0);
    float2* s_part = reinterpret_cast<float2*>(s_wk + (MODE == kModeFused ? p.dim : 0));

    const int tid = threadIdx.x;
    const int team = tid / p.tpr;
    const int t = tid - team * p.tpr;
    const int lane = tid & 31;
    const int warp_in_team = t >> 5;
    const int warps_per_team = p.tpr >> 5;

    if (MODE == kModeFused) {
        // Stage both weight vectors (dim is a multiple of 128, so float4 copies).
        const float4* gq = reinterpret_cast<const float4*>(p.q_w);
        const float4* gk = reinterpret_cast<const float4*>(p.k_w);
        float4* sq4 = reinterpret_cast<float4*>(s_wq);
        float4* sk4 = reinterpret_cast<float4*>(s_wk);
        for (int e = tid; e < p.dim / 4; e += blockDim.x) {
            sq4[e] = __ldg(gq + e);
            sk4[e] = __ldg(gk + e);
        }
        __syncthreads();
    }

    // The pairs this thread rotates: positions inside a head are fixed per thread.
    const int pair0 = (t % Tr::kVecsPerHead) * PPV;
    float inv[PPV];
    int axis[PPV];
    int tab_col[PPV];
#pragma unroll
    for (int m = 0; m < PPV; ++m) {
        const int j = pair0 + m;
        inv[m] = p.inv_freq[j];
        axis[m] = j < p.n_t ? 0 : (j < p.n_t + p.n_h ? 1 : 2);
        tab_col[m] = axis[m] == 0 ? j : (axis[m] == 1 ? j - p.n_t : j - p.n_t - p.n_h);
    }

    const Vec* qg = reinterpret_cast<const Vec*>(p.q);
    const Vec* kg = reinterpret_cast<const Vec*>(p.k);
    const Vec* vg = reinterpret_cast<const Vec*>(p.v);
    Vec* qo = reinterpret_cast<Vec*>(p.q_out);
    Vec* kc = reinterpret_cast<Vec*>(p.k_cache);
    Vec* vc = reinterpret_cast<Vec*>(p.v_cache);

    const int64_t stride = (int64_t)gridDim.x * p.teams;
    int parity = 0;
    for (int64_t u = (int64_t)blockIdx.x * p.teams + team; u < p.units; u += stride) {
        // ---- integer part: position decode (Section 3.3.3) and cache row
        const int64_t b = u / p.n_tok;
        const int64_t r = u - b * p.n_tok;
        const int64_t i = p.token_begin + r;
        const int64_t t_local = i / p.hw;
        const int64_t rem = i - t_local * p.hw;
        const int h = (int)(rem / p.W);
        const int w = (int)(rem - (int64_t)h * p.W);
        const int64_t t_g = p.frame_offset + t_local;

        // ---- loads (issued first, to keep many bytes in flight)
        const int64_t row_vec = u * p.dim_vecs;
        Vec xq[VPT], xk[VPT], xv[VPT];
#pragma unroll
        for (int s = 0; s < VPT; ++s) {
            const int idx = t + s * p.tpr;
            if (idx < p.dim_vecs) {
                xq[s] = load_stream(qg + row_vec + idx);
                if (MODE == kModeFused) {
                    xk[s] = load_stream(kg + row_vec + idx);
                    xv[s] = load_stream(vg + row_vec + idx);
                }
            }
        }

        // ---- cos / sin of this thread's pairs at (t_g, h, w)
        float cs[PPV], sn[PPV];
#pragma unroll
        for (int m = 0; m < PPV; ++m) {
            const int64_t pos = axis[m] == 0 ? t_g : (axis[m] == 1 ? (int64_t)h : (int64_t)w);
            if (TRIG == kTrigTable) {
                const float2* tab = axis[m] == 0 ? p.tab_t : (axis[m] == 1 ? p.tab_h : p.tab_w);
                const int ncol = axis[m] == 0 ? p.n_t : (axis[m] == 1 ? p.n_h : p.n_w);
                const float2 e = __ldg(tab + pos * ncol + tab_col[m]);
                cs[m] = e.x;
                sn[m] = e.y;
            } else {
                const float phi = (float)pos * inv[m];
                sincosf(phi, &sn[m], &cs[m]);
            }
        }

        float rq = 1.0f, rk = 1.0f;
        int64_t cache_vec = 0;
        if (MODE == kModeFused) {
            const int64_t crow = (p.slot + i) % p.cache_tokens;
            cache_vec = (b * p.cache_tokens + crow) * p.dim_vecs;
            // V goes to the cache untouched.
#pragma unroll
            for (int s = 0; s < VPT; ++s) {
                const int idx = t + s * p.tpr;
                if (idx < p.dim_vecs) store_out(vc + cache_vec + idx, xv[s]);
            }
            // Sum of squares of q and of k over the whole row, in a fixed order.
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int s = 0; s < VPT; ++s) {
                const int idx = t + s * p.tpr;
                if (idx < p.dim_vecs) {
#pragma unroll
                    for (int m = 0; m < PPV; ++m) {
                        float a, c;
                        Tr::pair(xq[s], m, a, c);
                        sq = fmaf(a, a, sq);
                        sq = fmaf(c, c, sq);
                        Tr::pair(xk[s], m, a, c);
                        sk = fmaf(a, a, sk);
                        sk = fmaf(c, c, sk);
                    }
                }
            }
            sq = warp_allreduce_sum(sq);
            sk = warp_allreduce_sum(sk);
            if (warps_per_team > 1) {
                float2* part = s_part + (parity * p.teams + team) * warps_per_team;
                if (lane == 0) part[warp_in_team] = make_float2(sq, sk);
                team_barrier(1 + team, p.tpr);
                sq = 0.f;
                sk = 0.f;
                for (int wi = 0; wi < warps_per_team; ++wi) {
                    const float2 pp = part[wi];
                    sq += pp.x;
                    sk += pp.y;
                }
                parity ^= 1;
            }
            rq = rsqrtf(fmaf(sq, p.inv_dim, p.eps));
            rk = rsqrtf(fmaf(sk, p.inv_dim, p.eps));
        }

        // ---- normalise, rotate, store
#pragma unroll
        for (int s = 0; s < VPT; ++s) {
            const int idx = t + s * p.tpr;
            if (idx < p.dim_vecs) {
                const int e0 = idx * EPV;
                Vec oq, ok;
#pragma unroll
                for (int m = 0; m < PPV; ++m) {
                    float a, c;
                    Tr::pair(xq[s], m, a, c);
                    if (MODE == kModeFused) {
                        const float2 wq = *reinterpret_cast<const float2*>(s_wq + e0 + 2 * m);
                        a = a * rq * wq.x;
                        c = c * rq * wq.y;
                    }
                    Tr::set_pair(oq, m, a * cs[m] - c * sn[m], a * sn[m] + c * cs[m]);
                    if (MODE == kModeFused) {
                        float ka, kb;
                        Tr::pair(xk[s], m, ka, kb);
                        const float2 wk = *reinterpret_cast<const float2*>(s_wk + e0 + 2 * m);
                        ka = ka * rk * wk.x;
                        kb = kb * rk * wk.y;
                        Tr::set_pair(ok, m, ka * cs[m] - kb * sn[m], ka * sn[m] + kb * cs[m]);
                    }
                }
                store_out(qo + row_vec + idx, oq);
                if (MODE == kModeFused) store_out(kc + cache_vec + idx, ok);
            }
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
