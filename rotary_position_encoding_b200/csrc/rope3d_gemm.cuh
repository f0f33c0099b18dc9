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
constexpr int kGemmGroupM = 32;
constexpr uint32_t kGemmStageA = kGemmBM * kGemmBK * 2;  // 16 KB
constexpr uint32_t kGemmStageB = kGemmBN * kGemmBK * 2;  // 32 KB
constexpr uint32_t kGemmTmemCols = 2 * kGemmBN;          // two accumulators
// dynamic shared memory: 1 KB alignment slack, the stages, then the barriers
constexpr size_t kGemmSmemBytes = 1024 + kGemmStages * (kGemmStageA + kGemmStageB) + 256;

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
    int* status;
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

__global__ void __launch_bounds__(kGemmThreads, 1)
qkv_proj_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                const GemmParams p) {
    extern __shared__ uint8_t gemm_smem_raw[];
    const uint32_t raw = smem_u32(gemm_smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 1 KB aligned: the swizzle atoms
    const uint32_t stage_a = base;
    const uint32_t stage_b = base + kGemmStages * kGemmStageA;
    const uint32_t bars = stage_b + kGemmStages * kGemmStageB;
    // barriers: full[S], empty[S], tmem_full[2], tmem_empty[2], drain; then the TMEM
    // address and the failure flag
    const uint32_t full_bar = bars, empty_bar = bars + 8 * kGemmStages;
    const uint32_t tfull_bar = bars + 16 * kGemmStages, tempty_bar = tfull_bar + 16;
    const uint32_t drain_bar = tempty_bar + 16;
    uint8_t* gen_base = gemm_smem_raw + (base - raw);
    const uint32_t bars_off = bars - base;
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(gen_base + bars_off + 128);
    volatile int* s_fail = reinterpret_cast<volatile int*>(gen_base + bars_off + 136);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.num_m * p.num_n;
    const int k_steps = p.K / kGemmBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(full_bar + 8 * s, 1);
            mbar_init(empty_bar + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar + 8 * a, 1);
            mbar_init(tempty_bar + 8 * a, 128);
        }
        mbar_init(drain_bar, 1);
        *s_fail = 0;
        fence_barrier_init();
    }
    if (warp == 1) {  // whole warp: allocate the accumulators' tensor memory
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32((const void*)s_tmem)), "r"(kGemmTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        if (lane == 0) {  // producer
            int s = 0, phase = 0;
            int armed = 0;  // stages armed and not yet known consumed (for the failure drain)
            for (int t = blockIdx.x; t < num_tiles && !*s_fail; t += gridDim.x) {
                int mb, nb;
                gemm_tile_coords(p, t, mb, nb);
                for (int kk = 0; kk < k_steps; ++kk) {
                    if (!mbar_wait_bounded(empty_bar + 8 * s, phase ^ 1, p.wait_limit_ns)) {
                        *s_fail = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(full_bar + 8 * s, kGemmStageA + kGemmStageB);
                    tma_load_2d(stage_a + s * kGemmStageA, &map_x, kk * kGemmBK, mb * kGemmBM,
                                full_bar + 8 * s);
                    tma_load_2d(stage_b + s * kGemmStageB, &map_w, kk * kGemmBK, nb * kGemmBN,
                                full_bar + 8 * s);
                    armed = min(armed + 1, kGemmStages);
                    if (++s == kGemmStages) { s = 0; phase ^= 1; }
                }
            }
            if (*s_fail) {  // let copies already issued land before the CTA can exit
                for (int j = 0; j < armed; ++j) {
                    if (--s < 0) { s = kGemmStages - 1; phase ^= 1; }
                    mbar_wait_bounded(full_bar + 8 * s, phase, p.wait_limit_ns);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // MMA issuer
            int s = 0, phase = 0, it = 0;
            for (int t = blockIdx.x; t < num_tiles && !*s_fail; t += gridDim.x, ++it) {
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
                    const uint64_t bdesc = smem_desc_sw128(stage_b + s * kGemmStageB);
#pragma unroll
                    for (int k = 0; k < kGemmBK / 16; ++k)  // 16 bf16 = 32 bytes along K
                        umma_bf16(d, adesc + 2 * k, bdesc + 2 * k, (kk | k) != 0);
                    umma_commit(empty_bar + 8 * s);  // the stage is free once these complete
                    if (++s == kGemmStages) { s = 0; phase ^= 1; }
                }
                if (*s_fail) break;
                umma_commit(tfull_bar + 8 * acc);
            }
            umma_commit(drain_bar);  // every tensor-core operation of this CTA is done
            mbar_wait_bounded(drain_bar, 0, p.wait_limit_ns);
        }
    } else {  // epilogue warps 2..5: lanes 32 (warp % 4) .. +32 of tensor memory
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        int it = 0;
        for (int t = blockIdx.x; t < num_tiles && !*s_fail; t += gridDim.x, ++it) {
            int mb, nb;
            gemm_tile_coords(p, t, mb, nb);
            const int acc = it & 1;
            const int use = it >> 1;
            if (!mbar_wait_bounded(tfull_bar + 8 * acc, use & 1, p.wait_limit_ns)) {
                *s_fail = 1;
                break;
            }
            tmem_fence_after();
            const int row = mb * kGemmBM + row_in_tile;
            const bool live = row < p.M;
            // destination of this row in the V cache
            int64_t v_row = 0;
            if (live) {
                const int64_t b = row / p.n_tok;
                const int64_t i = p.token_begin + (row - b * p.n_tok);
                const int64_t crow = (p.slot + i) % p.cache_tokens;
                v_row = p.cache_head_major ? (b * p.n_heads * p.cache_tokens + crow)
                                           : (b * p.cache_tokens + crow);
            }
            const uint32_t taddr = tmem + acc * kGemmBN + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
            for (int c = 0; c < kGemmBN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(taddr + c * 32, r);
                const int gc = nb * kGemmBN + c * 32;  // output column of the chunk
                if (!live || gc >= p.n_out) continue;
                const int which = gc / p.dim;         // 0 q, 1 k, 2 v
                const int col = gc - which * p.dim;
                uint32_t packed[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    float a = __uint_as_float(r[2 * j]), b = __uint_as_float(r[2 * j + 1]);
                    if (p.bias != nullptr) {
                        a += __ldg(p.bias + gc + 2 * j);
                        b += __ldg(p.bias + gc + 2 * j + 1);
                    }
                    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
                    packed[j] = *reinterpret_cast<uint32_t*>(&h);
                }
                __nv_bfloat16* dst;
                if (which == 0) {
                    dst = p.q_out + (int64_t)row * p.dim + col;
                } else if (which == 1) {
                    dst = p.k_out + (int64_t)row * p.dim + col;
                } else if (!p.cache_head_major) {
                    dst = p.v_cache + v_row * p.dim + col;
                } else {
                    const int head = col >> 7;
                    dst = p.v_cache + (v_row + (int64_t)head * p.cache_tokens) * 128 + (col & 127);
                }
                uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    d4[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                                       packed[4 * j + 3]);
            }
            tmem_fence_before();
            mbar_arrive(tempty_bar + 8 * acc);
        }
    }

    __syncwarp();  // the role lanes rejoin their warps
    tmem_fence_before();
    __syncthreads();
    if (*s_fail && threadIdx.x == 0 && p.status != nullptr) atomicExch(p.status, kStatusWaitTimeout);
    if (warp == 1) {
        tmem_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(kGemmTmemCols) : "memory");
    }
}

}  // namespace rope3d
