// rope3d_stream.cuh -- the fused step with token rows staged in shared memory by bulk
// asynchronous copies and consumed straight from there, for launches of few rows per SM
// (a 480P chunk, one sequence-parallel rank's slice) as well as long ones.
//
// One block per SM.  Warp 0 is the producer: its first lane keeps a ring of S stages
// (one token row of q, k and v each) filled with cp.async.bulk copies that complete on
// the stage's "full" mbarrier; it refills a stage once the team that consumed it has
// arrived on the stage's "empty" mbarrier.  The other warps form teams of TPR threads
// (the same team geometry as the other two kernels); team j consumes the block's rows
// j, j + T, j + 2T, ...  A team reads its row from the stage twice -- once for the
// RMSNorm sums, once to normalise, rotate and store -- so no thread holds a row in
// registers across the reduction.  That keeps registers low and lets S rows of the block
// be in flight at once: with small rows nearly a whole launch's loads are requested at
// its start.  The sums run in the same order as in the other kernels, so the results are
// bit-identical to them.
//
// Waits are bounded (p.wait_limit_ns): a team whose stage never fills leaves its loop
// after a vote at its reduction barrier and records kStatusWaitTimeout; the producer
// gives up on a stage that is never released, and before it returns waits (bounded) for
// every copy it issued to land.  No bulk copy uses cluster multicast.
#pragma once

#include "rope3d_tma.cuh"

namespace rope3d {

constexpr int kStreamMaxThreads = 640;  // one block per SM: up to 102 registers a thread

template <typename T, int VPT, int TRIG, int MODE, int PAIR, int CF>
__global__ void __launch_bounds__(kStreamMaxThreads, 1)
qk_norm_rope_stream_kernel(const Params p) {
    using Tr = VecTraits<T>;
    using Vec = typename Tr::Vec;
    constexpr int NP = PairCount<T, PAIR>::value;
    constexpr bool SP = MODE == kModeFusedSP;
    constexpr bool FP4 = CF == kCacheNvfp4;
    constexpr int STEP = PAIR == kPairHalf ? 2 : 1;  // slots handled together
    static_assert(MODE == kModeFused || MODE == kModeFusedSP, "fused step modes only");
    static_assert(!SP || (PAIR == kPairAdjacent && CF == kCacheSame),
                  "head-scatter stores: adjacent pairing, same-dtype caches");
    static_assert(VPT % STEP == 0, "rotate_half slots come in twos");

    // dynamic shared memory: [SP destination table | NVFP4 reciprocal tables] at 0, then
    // the full and empty barriers, the teams' failure flags and partial sums, the norm
    // weights and the stages (offsets from the host)
    extern __shared__ __align__(128) unsigned char smem[];
    void** s_sp = reinterpret_cast<void**>(smem);
    float* s_r = reinterpret_cast<float*>(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
    int* s_fail = reinterpret_cast<int*>(smem + p.off_fail);
    float2* s_part = reinterpret_cast<float2*>(smem + p.off_part);
    float* s_wq = reinterpret_cast<float*>(smem + p.off_w);
    float* s_wk = s_wq + p.dim;
    unsigned char* stage0 = smem + p.off_stage;

    const int tid = threadIdx.x;
    const int S = p.stages;
    const uint32_t rb = p.row_bytes;
    const uint32_t stage_bytes = 3u * rb;
    const uint32_t full0 = smem_u32(bars);
    const uint32_t empty0 = full0 + 8u * (uint32_t)S;
    const int64_t G = gridDim.x;
    // rows of this block: u = blockIdx.x + k G for k < rows (the grid is at most p.units)
    const int64_t rows = (p.units - 1 - (int64_t)blockIdx.x) / G + 1;

    // Arm stage (k mod S) for the block's k-th row and start its three copies.
    auto issue = [&](int64_t k) {
        const int s = (int)(k % S);
        const uint32_t bar = full0 + 8u * (uint32_t)s;
        const uint32_t dst = smem_u32(stage0) + (uint32_t)s * stage_bytes;
        const size_t off = (size_t)((int64_t)blockIdx.x + k * G) * rb;
        mbar_arrive_expect_tx(bar, stage_bytes + p.tx_extra);
        bulk_load(dst, static_cast<const char*>(p.q) + off, rb, bar);
        bulk_load(dst + rb, static_cast<const char*>(p.k) + off, rb, bar);
        bulk_load(dst + 2 * rb, static_cast<const char*>(p.v) + off, rb, bar);
    };

    pdl_launch_dependents();
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8u * s, 1);
            mbar_init(empty0 + 8u * s, (uint32_t)p.tpr);
        }
        for (int j = 0; j < p.teams; ++j) s_fail[j] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    pdl_wait_previous_grid();
    // The first rows are requested before the block stages its weights.
    const int64_t first = rows < S ? rows : S;
    if (tid == 0)
        for (int64_t k = 0; k < first; ++k) issue(k);
    if constexpr (SP) {
#pragma unroll
        for (int j = 0; j < 3 * kMaxRanks; ++j)
            if (tid == j) s_sp[j] = p.sp_dst[j];  // constant indices into the parameters
    }
    if constexpr (FP4) fill_nvfp4_tables(p, s_r);
    stage_weights(p, s_wq, s_wk);
    __syncthreads();

    if (tid < 32) {
        // ---- producer
        if (tid != 0) return;
        bool gave_up = false;
        int64_t k = first;
        for (; k < rows; ++k) {
            const int s = (int)(k % S);
            if (!mbar_wait_bounded(empty0 + 8u * s, (uint32_t)((k / S - 1) & 1),
                                   p.wait_limit_ns)) {
                gave_up = true;
                break;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(k);
        }
        if (gave_up) atomicOr(p.status, kStatusWaitTimeout);
        // every copy issued lands before the block's shared memory is released
        for (int64_t j = (k > S ? k - S : 0); j < k; ++j)
            mbar_wait_bounded(full0 + 8u * (uint32_t)(j % S), (uint32_t)((j / S) & 1),
                              p.wait_limit_ns);
        return;
    }

    // ---- consumer teams
    const int ct = tid - 32;
    const int team = ct / p.tpr;
    const int t = ct - team * p.tpr;
    if (team >= p.teams) return;
    const int lane = tid & 31;
    const int warp_in_team = t >> 5;
    const int warps_per_team = p.tpr >> 5;
    const PairInfo<NP> pi = pair_info<NP>(p, first_pair<T, PAIR>(t % Tr::kVecsPerHead));
    int dst[VPT];
    if constexpr (SP) {
#pragma unroll
        for (int s = 0; s < VPT; ++s) dst[s] = sp_code(p, slot_vec<T, PAIR>(t, s, p.tpr));
    }
    Vec* qo = reinterpret_cast<Vec*>(p.q_out);
    Vec* kc = reinterpret_cast<Vec*>(p.k_cache);
    Vec* vc = reinterpret_cast<Vec*>(p.v_cache);

    int parity = 0;
    bool failed = false;
    for (int64_t k = team; k < rows; k += p.teams) {
        const int s = (int)(k % S);
        const bool ok = mbar_wait_bounded(full0 + 8u * s, (uint32_t)((k / S) & 1),
                                          p.wait_limit_ns);
        const unsigned char* st = stage0 + (size_t)s * stage_bytes;
        const Vec* sq = reinterpret_cast<const Vec*>(st);
        const Vec* sk = reinterpret_cast<const Vec*>(st + rb);
        const Vec* sv = reinterpret_cast<const Vec*>(st + 2 * rb);

        // RMSNorm sums from the stage, in the other kernels' order
        float psq = 0.f, psk = 0.f;
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int idx = slot_vec<T, PAIR>(t, j, p.tpr);
            if (idx < p.dim_vecs) accumulate_squares(sq[idx], sk[idx], psq, psk);
        }
        // The reduction barrier is also the team's vote on a timed-out wait.
        if (!ok) s_fail[team] = 1;
        float2 tot;
        if (warps_per_team > 1) {
            tot = team_sum(psq, psk, s_part, team, p.teams, warp_in_team, warps_per_team, lane,
                           p.tpr, parity);
            failed = s_fail[team] != 0;
        } else {
            tot = team_sum(psq, psk, s_part, team, p.teams, 0, 1, lane, p.tpr, parity);
            failed = __any_sync(0xffffffffu, !ok);
        }
        if (failed) break;

        const int64_t u = (int64_t)blockIdx.x + k * G;
        const RowPos pos = decode_row(p, u);
        float cs[NP], sn[NP];
        pair_trig<TRIG>(p, pi, pos, cs, sn);
        const float rq = rsqrtf(fmaf(tot.x, p.inv_dim, p.eps));
        const float rk = rsqrtf(fmaf(tot.y, p.inv_dim, p.eps));
        const int64_t row_vec = u * p.dim_vecs;

        // normalise, rotate and store, STEP slots at a time, straight from the stage
#pragma unroll
        for (int j = 0; j < VPT; j += STEP) {
            // a thread whose slot j is slot 0 of "thread" t2 (see slot_vec)
            const int t2 = PAIR == kPairAdjacent ? t + j * p.tpr : t + (j >> 1) * p.tpr;
            Vec xq[STEP], xk[STEP], xv[STEP];
#pragma unroll
            for (int m = 0; m < STEP; ++m) {
                const int idx = slot_vec<T, PAIR>(t, j + m, p.tpr);
                if (idx < p.dim_vecs) {
                    xq[m] = sq[idx];
                    xk[m] = sk[idx];
                    xv[m] = sv[idx];
                }
            }
            if constexpr (SP) {
                const int d1[1] = {dst[j]};
                store_v_row_sp<T, 1>(p, t2, pos, xv, d1, s_sp);
                emit_row_sp<T, 1>(p, t2, pos, xq, xk, rq, rk, s_wq, s_wk, cs, sn, d1, s_sp);
            } else {
                if constexpr (CF == kCacheSame) store_v_row<T, STEP, PAIR>(p, t2, pos, xv, vc);
                emit_row<T, STEP, PAIR, kModeFused, CF>(p, t2, pos, row_vec, xq, xk, xv, rq, rk,
                                                        s_wq, s_wk, cs, sn, qo, kc, vc, s_r);
            }
        }
        mbar_arrive(empty0 + 8u * s);  // this thread is done with the stage
    }
    if (failed && t == 0) atomicOr(p.status, kStatusWaitTimeout);
}

}  // namespace rope3d
