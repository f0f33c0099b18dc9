// rope3d_tma.cuh -- the fused step with token rows streamed through shared memory by
// bulk asynchronous copies (cp.async.bulk, the 1-D form of the Tensor Memory
// Accelerator path) on sm_100a.
//
// Each team (see rope3d_kernels.cuh) owns a ring of S stages; a stage holds one token
// row of q, k and v (3 * N * 128 elements).  Thread 0 of the team is also the producer:
// it arms the stage's mbarrier with the byte count and issues three bulk copies, one
// per tensor.  The team waits on the mbarrier, copies its vectors from the stage into
// registers, and at the row's reduction barrier -- after which no thread reads the
// stage again -- the producer refills the stage with the row S ahead.  So S rows of
// every team are in flight from HBM regardless of the register budget.  Outputs go
// to global memory with ordinary 128-bit stores from registers.
//
// Waits are bounded: a stage that has not filled after p.wait_limit_ns makes the
// whole team (by a vote at the reduction barrier) leave its loop, record
// kStatusWaitTimeout in *p.status (read back as ROPE3D_ETIMEOUT), wait (bounded again)
// for its copies still in flight, and return.  No bulk copy uses cluster multicast.
#pragma once

#include "rope3d_kernels.cuh"

namespace rope3d {

constexpr int kStatusWaitTimeout = 1;

__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
    return (uint32_t)__cvta_generic_to_shared(ptr);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n"
        "  .reg .pred p;\n"
        "  mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "  selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// true once the barrier's phase of the given parity has completed; false after limit_ns
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// Global -> shared bulk copy completing on an mbarrier of this CTA (no multicast).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

template <typename T, int VPT, int TRIG, int PAIR, bool CFP8>
__global__ void __launch_bounds__(kTmaMaxBlockThreads, 1)
qk_norm_rope_tma_kernel(const Params p) {
    using Tr = VecTraits<T>;
    using Vec = typename Tr::Vec;
    constexpr int NP = PairCount<T, PAIR>::value;

    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
    int* s_fail = reinterpret_cast<int*>(smem + p.off_fail);
    float2* s_part = reinterpret_cast<float2*>(smem + p.off_part);
    float* s_wq = reinterpret_cast<float*>(smem + p.off_w);
    float* s_wk = s_wq + p.dim;

    const int tid = threadIdx.x;
    const int team = tid / p.tpr;
    const int t = tid - team * p.tpr;
    const int lane = tid & 31;
    const int warp_in_team = t >> 5;
    const int warps_per_team = p.tpr >> 5;
    const int S = p.stages;
    const uint32_t rb = p.row_bytes;
    const uint32_t stage_bytes = 3u * rb;
    unsigned char* ring = smem + p.off_stage + (size_t)team * S * stage_bytes;
    const uint32_t ring_u32 = smem_u32(ring);
    const uint32_t bar0 = smem_u32(bars + team * S);
    const int64_t G = (int64_t)gridDim.x * p.teams;       // teams in the grid
    const int64_t g = (int64_t)blockIdx.x * p.teams + team;  // this team's first row

    // Producer: arm stage (k mod S) for the team's k-th row and start its three copies.
    auto issue = [&](int64_t kk) {
        const int64_t u = g + kk * G;
        if (u >= p.units) return;
        const int s = (int)(kk % S);
        const uint32_t bar = bar0 + 8u * s;
        const uint32_t dst = ring_u32 + (uint32_t)s * stage_bytes;
        const size_t off = (size_t)u * rb;
        mbar_arrive_expect_tx(bar, stage_bytes + p.tx_extra);
        bulk_load(dst, static_cast<const char*>(p.q) + off, rb, bar);
        bulk_load(dst + rb, static_cast<const char*>(p.k) + off, rb, bar);
        bulk_load(dst + 2 * rb, static_cast<const char*>(p.v) + off, rb, bar);
    };

    pdl_launch_dependents();
    if (t == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bar0 + 8u * s, 1);
        s_fail[team] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    pdl_wait_previous_grid();
    // The first S rows are requested before the block stages its weights, so the two
    // latencies overlap at the start of the launch.
    if (t == 0)
        for (int kk = 0; kk < S; ++kk) issue(kk);
    stage_weights(p, s_wq, s_wk);
    __syncthreads();

    const PairInfo<NP> pi = pair_info<NP>(p, first_pair<T, PAIR>(t % Tr::kVecsPerHead));
    Vec* qo = reinterpret_cast<Vec*>(p.q_out);
    Vec* kc = reinterpret_cast<Vec*>(p.k_cache);
    Vec* vc = reinterpret_cast<Vec*>(p.v_cache);

    int parity = 0;
    int s = 0;            // stage of row k
    uint32_t phase = 0;   // parity of stage s's current use
    int64_t k = 0;
    bool failed = false;
    for (int64_t u = g; u < p.units; u += G, ++k) {
        const bool ok = mbar_wait_bounded(bar0 + 8u * s, phase, p.wait_limit_ns);
        const Vec* sq = reinterpret_cast<const Vec*>(ring + (size_t)s * stage_bytes);
        const Vec* sk = reinterpret_cast<const Vec*>(ring + (size_t)s * stage_bytes + rb);
        const Vec* sv = reinterpret_cast<const Vec*>(ring + (size_t)s * stage_bytes + 2 * rb);
        Vec xq[VPT], xk[VPT], xv[VPT];
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int idx = slot_vec<T, PAIR>(t, j, p.tpr);
            if (idx < p.dim_vecs) {
                xq[j] = sq[idx];
                xk[j] = sk[idx];
                xv[j] = sv[idx];
            }
        }
        float psq, psk;
        partial_sum_squares<T, VPT, PAIR>(xq, xk, t, p.tpr, p.dim_vecs, psq, psk);
        // The reduction barrier doubles as the team's "stage consumed" point and its
        // vote on a timed-out wait.
        if (!ok) s_fail[team] = 1;
        float2 tot;
        if (warps_per_team > 1) {
            tot = team_sum(psq, psk, s_part, team, p.teams, warp_in_team, warps_per_team, lane,
                           p.tpr, parity);
            failed = s_fail[team] != 0;
        } else {
            tot = team_sum(psq, psk, s_part, team, p.teams, 0, 1, lane, p.tpr, parity);
            failed = __any_sync(0xffffffffu, !ok);
            __syncwarp();
        }
        if (failed) break;
        if (t == 0) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(k + S);
        }
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }

        const RowPos pos = decode_row(p, u);
        float cs[NP], sn[NP];
        pair_trig<TRIG>(p, pi, pos, cs, sn);
        const float rq = rsqrtf(fmaf(tot.x, p.inv_dim, p.eps));
        const float rk = rsqrtf(fmaf(tot.y, p.inv_dim, p.eps));
        const int64_t row_vec = u * p.dim_vecs;
        if constexpr (!CFP8) store_v_row<T, VPT, PAIR>(p, t, pos, xv, vc);
        emit_row<T, VPT, PAIR, kModeFused, CFP8 ? kCacheFp8 : kCacheSame>(
            p, t, pos, row_vec, xq, xk, xv, rq, rk, s_wq, s_wk, cs, sn, qo, kc, vc);
    }

    if (failed && t == 0) {
        atomicOr(p.status, kStatusWaitTimeout);
        // Let the copies this team still has in flight land before the CTA's shared
        // memory is released: rows k .. k + S - 1 were issued (those below units).
        for (int64_t kk = k; kk < k + S; ++kk) {
            if (g + kk * G >= p.units) break;
            const int st = (int)(kk % S);
            const uint32_t ph = (uint32_t)((kk / S) & 1);
            mbar_wait_bounded(bar0 + 8u * st, ph, p.wait_limit_ns);
        }
    }
}

}  // namespace rope3d
