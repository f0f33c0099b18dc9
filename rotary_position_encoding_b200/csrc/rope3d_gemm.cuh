// rope3d_gemm.cuh -- the QKV projection that feeds the step (Algorithm 1/3 step 1 of
// "Accelerating Video Generation Inference with Sequential-Parallel 3D Positional Encoding
// Using a Global Time Index"; Section 3.4.1 item 3 fuses it with the rotary step) on the
// sm_100a tensor cores: y = x W^T + b with x [M][K] bf16 (token rows), W [3 dim][K] bf16
// (an nn.Linear weight: the q rows, then the k rows, then the v rows), fp32 accumulation
// in tensor memory, and an epilogue that rounds to bf16 and routes every 32-column chunk
// of a row to its destination: q to q_out (where the step then normalises and rotates it
// in place), k to a work buffer, and v straight into the V cache at the token's cache row
// (the append of Algorithm 1/3 step 5, fused here).
//
// One persistent CTA per SM, 6 warps:
//   warp 0      TMA producer: 128x64 tiles of x and 256x64 tiles of W (128-byte swizzle)
//               into a ring of kStages shared-memory stages, completing on mbarriers;
//   warp 1      allocates the 512 tensor-memory columns (two 128x256 fp32 accumulators)
//               and one elected lane issues tcgen05.mma (kind::f16, M=128 N=256 K=16)
//               for each stage, then tcgen05.commit to free the stage and, after a
//               tile's last stage, to hand the accumulator to the epilogue;
//   warps 2..5  epilogue: each thread owns one accumulator row (tensor-memory lane),
//               reads it 32 columns at a time (tcgen05.ld 32x32b.x32), adds the bias,
//               rounds to bf16 and stores; then frees the accumulator for the next tile.
// Tiles are visited in groups of kGroupM row blocks so that one wave of CTAs shares
// few distinct x and W tiles in L2.  Every mbarrier wait is bounded by p.wait_limit_ns;
// a role that gives up records kStatusWaitTimeout, every role then leaves its loop, the
// MMA warp waits (bounded) for its last tensor-core operations, and the tensor memory is
// released.  No copy uses cluster multicast.
#pragma once

#include <cuda.h>

#include "rope3d_tma.cuh"

namespace rope3d {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;   // 64 bf16 = 128 bytes: one swizzle row
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 192;
constexpr int kGemmGroupM = 16;
constexpr uint32_t kGemmStageA = kGemmBM * kGemmBK * 2;  // 16 KB
constexpr uint32_t kGemmStageB = kGemmBN * kGemmBK * 2;  // 32 KB
constexpr uint32_t kGemmTmemCols = 2 * kGemmBN;          // two accumulators
// Waits for work already issued (copies, tensor-core operations) before a CTA that gave up
// leaves: independent of the test-adjustable limit, so nothing is left in flight.
constexpr uint64_t kGemmDrainLimitNs = 250000000ull;  // 250 ms
// dynamic shared memory: 1 KB alignment slack, the stages, the barriers, and 16 KB that
// keeps every tensor-core operand read of the pair form inside the allocation
constexpr size_t kGemmSmemBytes =
    1024 + kGemmStages * (kGemmStageA + kGemmStageB) + 1024 + 16384;

struct GemmParams {
    int M;                 // token rows (B * n_tok)
    int K;                 // input features (multiple of 64)
    int n_out;             // 3 * dim (multiple of 128)
    int dim;               // N * 128
    int num_m, num_n;      // tiles
    const float* bias;     // [3 dim] fp32 or nullptr
    __nv_bfloat16* q_out;  // [M][dim]
    __nv_bfloat16* k_out;  // [M][dim]
    __nv_bfloat16* v_cache;  // [B][C][N][128] or [B][N][C][128]
    int64_t n_tok, token_begin, cache_tokens, slot;
    int n_heads;
    int cache_head_major;
    uint64_t wait_limit_ns;
    uint32_t tx_extra;         // extra bytes each stage waits for (0; tests use it to time out)
    int* status;
    // fused QK-RMSNorm + RoPE epilogue (dim a multiple of 256, so every tile is all q, all
    // k or all v): q and K tiles are stored weighted and rotated but not yet normalised,
    // with each row's partial sum of squares per tile; qk_row_scale_kernel then scales
    // every row by 1 / sqrt(mean + eps) in place.
    int fused;
    const float* q_w;          // [dim] RMSNorm weights
    const float* k_w;
    float eps, inv_dim;
    __nv_bfloat16* k_cache;    // [B][C][N][128] or [B][N][C][128]
    float* psum;               // [2][M][dim / 256] partial sums of squares
    const float2* tab_t;       // cos/sin tables, or null for on-the-fly fp32 sincos
    const float2* tab_h;
    const float2* tab_w;
    int n_t, n_h, n_w;
    int H, W;
    int64_t hw, frame_offset;
    float inv_freq[kPairs];
};

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major tile with the 128-byte swizzle: rows of
// 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), version 1, layout 2.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: bf16 A and B (K-major), fp32 D, M = 128, N = 256.
constexpr uint32_t kGemmIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                ((uint32_t)(kGemmBN >> 3) << 17) |
                                ((uint32_t)(kGemmBM >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kGemmIdesc), "r"(accumulate)
        : "memory");
}

// Arrive on a CTA mbarrier once every tensor-core operation issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Barrier 1 over the 4 epilogue warps, with the OR / AND of a predicate: every epilogue
// thread gets the same answer, so the group always takes the same branch.
__device__ __forceinline__ bool epi_vote_any(bool v) {
    uint32_t r;
    asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
                 " bar.red.or.pred q, 1, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
                 : "=r"(r) : "r"((uint32_t)v) : "memory");
    return r != 0;
}
__device__ __forceinline__ bool epi_vote_all(bool v) {
    uint32_t r;
    asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
                 " bar.red.and.pred q, 1, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
                 : "=r"(r) : "r"((uint32_t)v) : "memory");
    return r != 0;
}

// ---- the pair form (cta_group::2): two CTAs of a cluster share each 256x256 tile; each
// holds 128 rows of x and 128 rows of W per stage and 128 accumulator rows, and the even
// CTA issues the tensor-core operations for both.
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// The address of this CTA's shared-memory word `addr` in cluster CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.aligned;\nbarrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
                 ::"r"(cluster_addr) : "memory");
}
// 2-D TMA load into this CTA's shared memory completing on a barrier of either CTA of the
// pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x,
                                                 int y, uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}
// Instruction descriptor of the pair form: M = 256 across the two CTAs, N = 256.
constexpr uint32_t kGemmIdescPair = (1u << 4) | (1u << 7) | (1u << 10) |
                                    ((uint32_t)(kGemmBN >> 3) << 17) |
                                    ((uint32_t)(2 * kGemmBM >> 4) << 24);
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kGemmIdescPair), "r"(accumulate)
        : "memory");
}
// Arrive on the barrier at this offset in both CTAs of the pair once the pair's
// tensor-core operations issued so far have completed.
__device__ __forceinline__ void umma_commit_pair_both(uint32_t bar) {
    asm volatile(
        "{\n .reg .b16 m;\n mov.b16 m, 3;\n"
        " tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n}" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        ::"r"(bar) : "memory");
}

template <int G> struct GemmShape {
    static constexpr int kStages = G == 1 ? kGemmStages : 6;
    static constexpr uint32_t kStageB = (kGemmBN / G) * kGemmBK * 2;  // this CTA's W rows
    static constexpr int kTileM = kGemmBM * G;                       // rows of a tile
};

// Tile t -> (row block, column block), grouped kGemmGroupM row blocks at a time.
__device__ __forceinline__ void gemm_tile_coords(const GemmParams& p, int t, int& mb, int& nb) {
    const int per_group = kGemmGroupM * p.num_n;
    const int g = t / per_group;
    const int first = g * kGemmGroupM;
    const int rows = min(kGemmGroupM, p.num_m - first);
    const int r = t - g * per_group;
    mb = first + r % rows;
    nb = r / rows;
}

template <int G>
__global__ void __launch_bounds__(kGemmThreads, 1)
qkv_proj_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                const GemmParams p) {
    constexpr int STAGES = GemmShape<G>::kStages;
    constexpr uint32_t STAGE_B = GemmShape<G>::kStageB;
    constexpr int TILE_M = GemmShape<G>::kTileM;
    extern __shared__ uint8_t gemm_smem_raw[];
    const uint32_t raw = smem_u32(gemm_smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 1 KB aligned: the swizzle atoms
    const uint32_t stage_a = base;
    const uint32_t stage_b = base + STAGES * kGemmStageA;
    const uint32_t bars = stage_b + STAGES * STAGE_B;
    // barriers: full[S], empty[S], tmem_full[2], tmem_empty[2], drain; then the TMEM
    // address and the failure flag
    const uint32_t full_bar = bars, empty_bar = bars + 8 * STAGES;
    const uint32_t tfull_bar = bars + 16 * STAGES, tempty_bar = tfull_bar + 16;
    const uint32_t drain_bar = tempty_bar + 16;
    const uint32_t rank = G == 2 ? cluster_rank() : 0;
    const int first_tile = G == 2 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int tile_stride = G == 2 ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    uint8_t* gen_base = gemm_smem_raw + (base - raw);
    const uint32_t bars_off = bars - base;
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(gen_base + bars_off + 256);
    volatile int* s_fail = reinterpret_cast<volatile int*>(gen_base + bars_off + 264);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.num_m * p.num_n;
    const int k_steps = p.K / kGemmBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar + 8 * s, 1);
            mbar_init(empty_bar + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar + 8 * a, 1);
            mbar_init(tempty_bar + 8 * a, 128 * G);  // the epilogue threads of every CTA
        }
        mbar_init(drain_bar, 1);
        *s_fail = 0;
        fence_barrier_init();
    }
    if (warp == 1) {  // whole warp: allocate the accumulators' tensor memory
        if constexpr (G == 1) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32((const void*)s_tmem)), "r"(kGemmTmemCols) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32((const void*)s_tmem)), "r"(kGemmTmemCols) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        }
    }
    tmem_fence_before();
    __syncthreads();
    if constexpr (G == 2) cluster_sync();  // both CTAs' barriers exist before any use
    tmem_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        if (lane == 0) {  // producer
            int s = 0, phase = 0;
            int armed = 0;  // stages armed and not yet known consumed (for the failure drain)
            for (int t = first_tile; t < num_tiles && !*s_fail; t += tile_stride) {
                int mb, nb;
                gemm_tile_coords(p, t, mb, nb);
                for (int kk = 0; kk < k_steps; ++kk) {
                    if (!mbar_wait_bounded(empty_bar + 8 * s, phase ^ 1, p.wait_limit_ns)) {
                        *s_fail = 1;
                        break;
                    }
                    if constexpr (G == 1) {
                        mbar_arrive_expect_tx(full_bar + 8 * s,
                                              kGemmStageA + STAGE_B + p.tx_extra);
                        tma_load_2d(stage_a + s * kGemmStageA, &map_x, kk * kGemmBK,
                                    mb * kGemmBM, full_bar + 8 * s);
                        tma_load_2d(stage_b + s * STAGE_B, &map_w, kk * kGemmBK, nb * kGemmBN,
                                    full_bar + 8 * s);
                    } else {
                        // both CTAs' copies complete on the even CTA's barrier, which
                        // expects the pair's bytes
                        const uint32_t bar = map_to_rank(full_bar + 8 * s, 0);
                        if (rank == 0)
                            mbar_arrive_expect_tx(full_bar + 8 * s,
                                                  2 * (kGemmStageA + STAGE_B) + p.tx_extra);
                        tma_load_2d_pair(stage_a + s * kGemmStageA, &map_x, kk * kGemmBK,
                                         mb * TILE_M + (int)rank * kGemmBM, bar);
                        tma_load_2d_pair(stage_b + s * STAGE_B, &map_w, kk * kGemmBK,
                                         nb * kGemmBN + (int)rank * (kGemmBN / 2), bar);
                    }
                    armed = min(armed + 1, STAGES);
                    if (++s == STAGES) { s = 0; phase ^= 1; }
                }
            }
            if (*s_fail && (G == 1 || rank == 0)) {  // let copies already issued land
                for (int j = 0; j < armed; ++j) {
                    if (--s < 0) { s = STAGES - 1; phase ^= 1; }
                    mbar_wait_bounded(full_bar + 8 * s, phase, kGemmDrainLimitNs);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {  // MMA issuer (the even CTA of a pair)
            int s = 0, phase = 0, it = 0;
            for (int t = first_tile; t < num_tiles && !*s_fail; t += tile_stride, ++it) {
                const int acc = it & 1;
                const int use = it >> 1;  // how many times this accumulator was used before
                if (!mbar_wait_bounded(tempty_bar + 8 * acc, (use & 1) ^ 1, p.wait_limit_ns)) {
                    *s_fail = 1;
                    break;
                }
                tmem_fence_after();
                const uint32_t d = tmem + acc * kGemmBN;
                for (int kk = 0; kk < k_steps; ++kk) {
                    if (!mbar_wait_bounded(full_bar + 8 * s, phase, p.wait_limit_ns)) {
                        *s_fail = 1;
                        break;
                    }
                    tmem_fence_after();
                    const uint64_t adesc = smem_desc_sw128(stage_a + s * kGemmStageA);
                    const uint64_t bdesc = smem_desc_sw128(stage_b + s * STAGE_B);
#pragma unroll
                    for (int k = 0; k < kGemmBK / 16; ++k) {  // 16 bf16 = 32 bytes along K
                        if constexpr (G == 1)
                            umma_bf16(d, adesc + 2 * k, bdesc + 2 * k, (kk | k) != 0);
                        else
                            umma_bf16_pair(d, adesc + 2 * k, bdesc + 2 * k, (kk | k) != 0);
                    }
                    // the stage is free (in every CTA) once these complete
                    if constexpr (G == 1) umma_commit(empty_bar + 8 * s);
                    else umma_commit_pair_both(empty_bar + 8 * s);
                    if (++s == STAGES) { s = 0; phase ^= 1; }
                }
                if (*s_fail) break;
                if constexpr (G == 1) umma_commit(tfull_bar + 8 * acc);
                else umma_commit_pair_both(tfull_bar + 8 * acc);
            }
            // every tensor-core operation of this CTA (pair) is done
            if constexpr (G == 1) umma_commit(drain_bar);
            else umma_commit_pair(drain_bar);
            mbar_wait_bounded(drain_bar, 0, kGemmDrainLimitNs);
        }
    } else {  // epilogue warps 2..5: lanes 32 (warp % 4) .. +32 of tensor memory
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        const int tiles_per_tensor = p.dim / kGemmBN;
        int it = 0;
        for (int t = first_tile; t < num_tiles; t += tile_stride, ++it) {
            if (epi_vote_any(*s_fail != 0)) break;  // the group leaves together
            int mb, nb;
            gemm_tile_coords(p, t, mb, nb);
            const int acc = it & 1;
            const int use = it >> 1;
            const bool got = mbar_wait_bounded(tfull_bar + 8 * acc, use & 1, p.wait_limit_ns);
            if (!epi_vote_all(got)) {
                *s_fail = 1;
                break;
            }
            tmem_fence_after();
            const int row = mb * TILE_M + (int)rank * kGemmBM + row_in_tile;
            const bool live = row < p.M;
            const int which_tile = (nb * kGemmBN) / p.dim;  // 0 q, 1 k, 2 v (fused layout)
            const bool norm_tile = p.fused && which_tile < 2;
            // this row's token: batch b, index i, position and cache row
            int64_t b = 0, i = 0, crow = 0, t_g = 0;
            int hh = 0, ww = 0;
            if (live) {
                b = row / p.n_tok;
                i = p.token_begin + (row - b * p.n_tok);
                crow = (p.slot + i) % p.cache_tokens;
                if (norm_tile) {
                    const int64_t tl = i / p.hw;
                    const int64_t rem = i - tl * p.hw;
                    t_g = p.frame_offset + tl;
                    hh = (int)(rem / p.W);
                    ww = (int)(rem - (int64_t)hh * p.W);
                }
            }
            const int64_t v_row = p.cache_head_major ? (b * p.n_heads * p.cache_tokens + crow)
                                                     : (b * p.cache_tokens + crow);
            const uint32_t taddr = tmem + acc * kGemmBN + ((uint32_t)(quarter * 32) << 16);
            float ss = 0.0f;  // this row's sum of squares over the tile (fixed order)
#pragma unroll 1
            for (int c = 0; c < kGemmBN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(taddr + c * 32, r);
                const int gc = nb * kGemmBN + c * 32;  // output column of the chunk
                if (!live || gc >= p.n_out) continue;
                const int which = gc / p.dim;         // 0 q, 1 k, 2 v
                const int col = gc - which * p.dim;
                float a[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) a[j] = __uint_as_float(r[j]);
                if (p.bias != nullptr) {  // 32 consecutive fp32: 8 aligned 16-byte loads
                    const float4* b4 = reinterpret_cast<const float4*>(p.bias + gc);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 bb = __ldg(b4 + q);
                        a[4 * q] += bb.x;
                        a[4 * q + 1] += bb.y;
                        a[4 * q + 2] += bb.z;
                        a[4 * q + 3] += bb.w;
                    }
                }
                uint32_t packed[16];
                if (norm_tile) {
                    // every load of the chunk is issued before the arithmetic: the weights
                    // (8 aligned 16-byte loads) and the 16 (cos, sin) pairs, whose table and
                    // row are chosen without branches
                    const float4* w4 =
                        reinterpret_cast<const float4*>((which == 0 ? p.q_w : p.k_w) + col);
                    float wv[32];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 t4 = __ldg(w4 + q);
                        wv[4 * q] = t4.x;
                        wv[4 * q + 1] = t4.y;
                        wv[4 * q + 2] = t4.z;
                        wv[4 * q + 3] = t4.w;
                    }
                    const int pair0 = (col & 127) >> 1;  // first pair of the chunk in its head
                    float cs[16], sn[16];
                    if (p.tab_t != nullptr) {
                        float2 e[16];
#pragma unroll
                        for (int m = 0; m < 16; ++m) {
                            const int j = pair0 + m;
                            const bool in_t = j < p.n_t, in_h = !in_t && j < p.n_t + p.n_h;
                            const float2* tab = in_t ? p.tab_t : (in_h ? p.tab_h : p.tab_w);
                            const int64_t at = in_t ? t_g * p.n_t + j
                                               : in_h ? (int64_t)hh * p.n_h + (j - p.n_t)
                                                      : (int64_t)ww * p.n_w + (j - p.n_t - p.n_h);
                            e[m] = __ldg(tab + at);
                        }
#pragma unroll
                        for (int m = 0; m < 16; ++m) {
                            cs[m] = e[m].x;
                            sn[m] = e[m].y;
                        }
                    } else {
#pragma unroll
                        for (int m = 0; m < 16; ++m) {
                            const int j = pair0 + m;
                            const int64_t x = j < p.n_t ? t_g : (j < p.n_t + p.n_h ? hh : ww);
                            sincosf((float)x * p.inv_freq[j], &sn[m], &cs[m]);
                        }
                    }
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        ss = fmaf(a[2 * m], a[2 * m], ss);
                        ss = fmaf(a[2 * m + 1], a[2 * m + 1], ss);
                        const float x0 = a[2 * m] * wv[2 * m];
                        const float x1 = a[2 * m + 1] * wv[2 * m + 1];
                        __nv_bfloat162 h = __floats2bfloat162_rn(x0 * cs[m] - x1 * sn[m],
                                                                 x0 * sn[m] + x1 * cs[m]);
                        packed[m] = *reinterpret_cast<uint32_t*>(&h);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(a[2 * j], a[2 * j + 1]);
                        packed[j] = *reinterpret_cast<uint32_t*>(&h);
                    }
                }
                __nv_bfloat16* dst;
                const int head = col >> 7;
                if (which == 0) {
                    dst = p.q_out + (int64_t)row * p.dim + col;
                } else if (which == 1 && !p.fused) {
                    dst = p.k_out + (int64_t)row * p.dim + col;
                } else {
                    __nv_bfloat16* cache = which == 1 ? p.k_cache : p.v_cache;
                    dst = !p.cache_head_major
                              ? cache + v_row * p.dim + col
                              : cache + (v_row + (int64_t)head * p.cache_tokens) * 128 + (col & 127);
                }
                uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    d4[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                                       packed[4 * j + 3]);
            }
            tmem_fence_before();
            // the accumulator is free for the next tile (the even CTA's barrier counts both)
            if constexpr (G == 1) mbar_arrive(tempty_bar + 8 * acc);
            else mbar_arrive_cluster(map_to_rank(tempty_bar + 8 * acc, 0));
            // record this row's partial sum of squares over the tile's columns
            if (norm_tile && live) {
                const int tile_in_tensor = nb - which_tile * tiles_per_tensor;
                p.psum[((int64_t)which_tile * p.M + row) * tiles_per_tensor + tile_in_tensor] = ss;
            }
        }
    }

    __syncwarp();  // the role lanes rejoin their warps
    tmem_fence_before();
    __syncthreads();
    // the pair stays resident until the even CTA's last operations on the odd CTA's
    // shared memory and barriers are done
    if constexpr (G == 2) cluster_sync();
    if (*s_fail && threadIdx.x == 0 && p.status != nullptr) atomicExch(p.status, kStatusWaitTimeout);
    if (warp == 1) {
        tmem_fence_after();
        if constexpr (G == 1)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                         ::"r"(tmem), "r"(kGemmTmemCols) : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
                         ::"r"(tmem), "r"(kGemmTmemCols) : "memory");
    }
}

// The normalisation that completes the fused epilogue: one warp per (tensor, row) sums
// the row's partial sums of squares (lane-strided, then a butterfly: a fixed order, so
// slices and wholes agree bit for bit) and scales the row's dim bf16 values -- q in q_out,
// K in its cache row -- by 1 / sqrt(mean + eps) in place, 16 bytes per lane and access,
// kScaleUnroll accesses in flight per lane.
constexpr int kScaleWarps = 8;
constexpr int kScaleUnroll = 4;

__global__ void __launch_bounds__(32 * kScaleWarps)
qk_row_scale_kernel(const GemmParams p) {
    pdl_launch_dependents();
    pdl_wait_previous_grid();
    const int task = blockIdx.x * kScaleWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (task >= 2 * p.M) return;
    const int which = task >= p.M ? 1 : 0;  // 0 q, 1 K
    const int row = task - which * p.M;
    const int tiles = p.dim / kGemmBN;
    const float* ps = p.psum + ((int64_t)which * p.M + row) * tiles;
    float part = 0.0f;
    for (int k = lane; k < tiles; k += 32) part += __ldg(ps + k);
    const float rs = rsqrtf(fmaf(warp_allreduce_sum(part), p.inv_dim, p.eps));
    const int64_t b = row / p.n_tok;
    const int64_t i = p.token_begin + (row - b * p.n_tok);
    const int64_t crow = (p.slot + i) % p.cache_tokens;
    const int vpr = p.dim / 8;
    for (int v0 = lane; v0 < vpr; v0 += 32 * kScaleUnroll) {
        uint4* ptr[kScaleUnroll];
        uint4 x[kScaleUnroll];
#pragma unroll
        for (int u = 0; u < kScaleUnroll; ++u) {
            const int v = v0 + 32 * u;
            ptr[u] = nullptr;
            if (v < vpr) {
                const int col = v * 8;
                ptr[u] = reinterpret_cast<uint4*>(
                    which == 0 ? p.q_out + (int64_t)row * p.dim + col
                    : !p.cache_head_major
                        ? p.k_cache + (b * p.cache_tokens + crow) * p.dim + col
                        : p.k_cache + ((b * p.n_heads + (col >> 7)) * p.cache_tokens + crow) * 128 +
                              (col & 127));
                x[u] = __ldcs(ptr[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < kScaleUnroll; ++u) {
            if (ptr[u] == nullptr) continue;
            uint32_t* w4 = reinterpret_cast<uint32_t*>(&x[u]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w4[q]);
                const float2 f = __bfloat1622float2(h);
                h = __floats2bfloat162_rn(f.x * rs, f.y * rs);
                w4[q] = *reinterpret_cast<uint32_t*>(&h);
            }
            __stcs(ptr[u], x[u]);
        }
    }
}

}  // namespace rope3d
