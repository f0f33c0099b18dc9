// rope3d.cu -- host side of librope3d.so: argument checks, frequency tables and
// kernel launches behind the C ABI of include/rope3d.h.
//
// Paper: "Accelerating Video Generation Inference with Sequential-Parallel 3D
// Positional Encoding Using a Global Time Index" (Yuan & Li).  The tables follow
// Section 3.4.1 item 2 (precomputed contiguous cos/sin tensors instead of a per-call
// cache) and Algorithm 2 (one table per axis, concatenated t | h | w).
#include "rope3d.h"
#include "rope3d_testing.h"
#include "rope3d_kernels.cuh"
#include "rope3d_tma.cuh"
#include "rope3d_gemm.cuh"

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#ifndef ROPE3D_VPT_TARGET
#define ROPE3D_VPT_TARGET 4  // vectors per thread per tensor the team size aims for
#endif
#ifndef ROPE3D_MAX_VPT
#define ROPE3D_MAX_VPT 4     // kernels are instantiated for 1 .. ROPE3D_MAX_VPT vectors
#endif
// Threads per block the team count aims for, per kernel path.  Measured on B200 at the
// 720P shape (40 heads, TPR 160): the register kernel is fastest with one team per
// block (several blocks per SM); the bulk-copy ring with two teams of three stages.
#ifndef ROPE3D_REG_BLOCK_TARGET
#define ROPE3D_REG_BLOCK_TARGET 256
#endif
#ifndef ROPE3D_TMA_BLOCK_TARGET
#define ROPE3D_TMA_BLOCK_TARGET 320
#endif
// Output all-to-all: units per thread per step, and whether 32-byte units are used when
// the pointers allow them.
#ifndef ROPE3D_A2A_UNROLL
#define ROPE3D_A2A_UNROLL 2
#endif
#ifndef ROPE3D_A2A_WIDE
#define ROPE3D_A2A_WIDE 1
#endif

struct rope3d_tables {
    int device;
    int head_dim;
    int n_t, n_h, n_w;
    double theta;
    int schedule;
    int max_t, max_h, max_w;
    float2* d_tab;  // one allocation: t table, then h, then w
    float2* tab_t;
    float2* tab_h;
    float2* tab_w;
    int* d_status;  // device word the bounded waits of the TMA kernel report into
    float inv_freq[rope3d::kPairs];
};

namespace {

thread_local char g_last_error[512] = "";

// Settings that tests use to exercise the bounded waits and both kernel paths.
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};
std::atomic<uint32_t> g_tx_extra{0};
std::atomic<int> g_force_path{ROPE3D_PATH_AUTO};
std::atomic<int> g_gemm_cta_group{2};  // the projection's form: 1 CTA or a 2-CTA pair per tile
std::atomic<int64_t> g_check_shrink{0};  // checked build: cache rows the row check withholds
thread_local int g_last_path = ROPE3D_PATH_AUTO;  // path of this thread's last fused launch

int fail(int status, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return status;
}

int ok() {
    g_last_error[0] = '\0';
    return ROPE3D_OK;
}

// ---- per-device facts, looked up once
struct DeviceInfo {
    bool known = false;
    bool supported = false;
    int sms = 0;
    int max_smem_optin = 0;
};
std::mutex g_mutex;
std::vector<DeviceInfo> g_devices;

int device_info(DeviceInfo* out, int* device) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    std::lock_guard<std::mutex> lock(g_mutex);
    if ((int)g_devices.size() <= dev) g_devices.resize(dev + 1);
    DeviceInfo& d = g_devices[dev];
    if (!d.known) {
        int major = 0, minor = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) ||
            (e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) ||
            (e = cudaDeviceGetAttribute(&d.max_smem_optin,
                                        cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)))
            return fail(ROPE3D_ECUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        d.supported = (major == 10 && minor == 0);
        d.known = true;
    }
    if (!d.supported)
        return fail(ROPE3D_EDEVICE, "device %d is not compute capability 10.0 (sm_100a)", dev);
    *out = d;
    *device = dev;
    return ROPE3D_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// Checks shared by the fused and apply entry points.
int check_common(int64_t B, int64_t N, int D, int dtype, int64_t token_begin,
                 int64_t token_end, int64_t frame_offset, int T, int H, int W,
                 const rope3d_tables* tables, int trig) {
    if (tables == nullptr) return fail(ROPE3D_EINVAL, "tables is NULL");
    if (dtype != ROPE3D_F32 && dtype != ROPE3D_BF16)
        return fail(ROPE3D_EINVAL, "dtype %d is neither ROPE3D_F32 nor ROPE3D_BF16", dtype);
    if (D != rope3d::kHeadDim || D != tables->head_dim)
        return fail(ROPE3D_EINVAL, "head size D=%d: the kernels and these tables need %d", D,
                    tables->head_dim);
    if (B < 1 || N < 1) return fail(ROPE3D_EINVAL, "B=%lld and N=%lld must be >= 1",
                                    (long long)B, (long long)N);
    if (T < 1 || H < 1 || W < 1)
        return fail(ROPE3D_EINVAL, "grid T=%d H=%d W=%d must be >= 1", T, H, W);
    if (frame_offset < 0) return fail(ROPE3D_EINVAL, "frame_offset %lld < 0",
                                      (long long)frame_offset);
    const int64_t L = (int64_t)T * H * W;
    if (token_begin < 0 || token_end <= token_begin)
        return fail(ROPE3D_ERANGE, "token range [%lld, %lld) is empty or negative",
                    (long long)token_begin, (long long)token_end);
    if (token_end > L)
        return fail(ROPE3D_ERANGE, "token_end %lld exceeds T*H*W = %lld", (long long)token_end,
                    (long long)L);
    if (trig != ROPE3D_TRIG_TABLE && trig != ROPE3D_TRIG_ONTHEFLY)
        return fail(ROPE3D_EINVAL, "trig %d is not a ROPE3D_TRIG_* value", trig);
    if (trig == ROPE3D_TRIG_TABLE) {
        const int64_t t_last = frame_offset + (token_end - 1) / ((int64_t)H * W);
        if (tables->d_tab == nullptr)
            return fail(ROPE3D_ERANGE, "these tables hold no cos/sin rows; use ROPE3D_TRIG_ONTHEFLY");
        if (t_last >= tables->max_t || H > tables->max_h || W > tables->max_w)
            return fail(ROPE3D_ERANGE,
                        "positions exceed the tables: frame %lld (max_t %d), H %d (max_h %d), "
                        "W %d (max_w %d)", (long long)t_last, tables->max_t, H, tables->max_h,
                        W, tables->max_w);
    }
    return ROPE3D_OK;
}

// Team geometry, a function of (N, dtype, pairing) only -- it fixes the reduction order,
// so it must not depend on the token range or the grid.
struct Geometry {
    int dim_vecs;
    int tpr;
    int vpt;
};

Geometry geometry(int64_t N, int dtype, int pairing) {
    const int elems_per_vec = dtype == ROPE3D_BF16 ? 8 : 4;
    Geometry g;
    g.dim_vecs = (int)(N * rope3d::kHeadDim / elems_per_vec);
    if (pairing == ROPE3D_PAIRING_HALF) {
        // slots come in twos (a head's two halves at one position): count half units
        const int units = g.dim_vecs / 2;
        const int per_warp = 32 * (ROPE3D_VPT_TARGET / 2);
        g.tpr = 32 * ((units + per_warp - 1) / per_warp);
        g.vpt = 2 * ((units + g.tpr - 1) / g.tpr);
        return g;
    }
    const int per_warp = 32 * ROPE3D_VPT_TARGET;
    g.tpr = 32 * ((g.dim_vecs + per_warp - 1) / per_warp);
    g.vpt = (g.dim_vecs + g.tpr - 1) / g.tpr;
    return g;
}

using KernelFn = void (*)(const rope3d::Params);

// Kernel instantiation for the launch's element type, trig mode, pairing, cache format
// and vectors per thread.  Pairing rotate_half uses even VPT only (slots come in twos);
// the rotation-only mode writes no cache.

template <typename T, int TRIG, int MODE, int PAIR, int CF>
KernelFn pick_vpt(int vpt) {
    if constexpr (PAIR == rope3d::kPairHalf) {
        switch (vpt) {
            case 2: return rope3d::qk_norm_rope_kernel<T, 2, TRIG, MODE, PAIR, CF>;
            case 4: return rope3d::qk_norm_rope_kernel<T, 4, TRIG, MODE, PAIR, CF>;
#if ROPE3D_MAX_VPT >= 6
            case 6: return rope3d::qk_norm_rope_kernel<T, 6, TRIG, MODE, PAIR, CF>;
#endif
            default: return nullptr;
        }
    } else {
        switch (vpt) {
            case 1: return rope3d::qk_norm_rope_kernel<T, 1, TRIG, MODE, PAIR, CF>;
            case 2: return rope3d::qk_norm_rope_kernel<T, 2, TRIG, MODE, PAIR, CF>;
            case 3: return rope3d::qk_norm_rope_kernel<T, 3, TRIG, MODE, PAIR, CF>;
            case 4: return rope3d::qk_norm_rope_kernel<T, 4, TRIG, MODE, PAIR, CF>;
#if ROPE3D_MAX_VPT >= 6
            case 5: return rope3d::qk_norm_rope_kernel<T, 5, TRIG, MODE, PAIR, CF>;
            case 6: return rope3d::qk_norm_rope_kernel<T, 6, TRIG, MODE, PAIR, CF>;
#endif
            default: return nullptr;
        }
    }
}

template <typename T, int MODE, int PAIR, int CF>
KernelFn pick_trig(int trig, int vpt) {
    return trig == ROPE3D_TRIG_TABLE ? pick_vpt<T, rope3d::kTrigTable, MODE, PAIR, CF>(vpt)
                                     : pick_vpt<T, rope3d::kTrigOnTheFly, MODE, PAIR, CF>(vpt);
}

template <typename T, int MODE, int CF>
KernelFn pick_pairing(int pairing, int trig, int vpt) {
    return pairing == ROPE3D_PAIRING_HALF ? pick_trig<T, MODE, rope3d::kPairHalf, CF>(trig, vpt)
                                          : pick_trig<T, MODE, rope3d::kPairAdjacent, CF>(trig, vpt);
}

template <typename T, int MODE>
KernelFn pick_format(int cache_fmt, int pairing, int trig, int vpt) {
    switch (cache_fmt) {
        case rope3d::kCacheFp8: return pick_pairing<T, MODE, rope3d::kCacheFp8>(pairing, trig, vpt);
        case rope3d::kCacheNvfp4:
            return pick_pairing<T, MODE, rope3d::kCacheNvfp4>(pairing, trig, vpt);
        default: return pick_pairing<T, MODE, rope3d::kCacheSame>(pairing, trig, vpt);
    }
}

template <int MODE>
KernelFn pick_kernel(int dtype, int trig, int pairing, int cache_fmt, int vpt) {
    if constexpr (MODE == rope3d::kModeFusedNoV) {
        // the step after the QKV projection: bf16, adjacent pairing, same-dtype K cache
        if (pairing != ROPE3D_PAIRING_ADJACENT || cache_fmt != rope3d::kCacheSame ||
            dtype != ROPE3D_BF16)
            return nullptr;
        return pick_trig<__nv_bfloat16, MODE, rope3d::kPairAdjacent, rope3d::kCacheSame>(trig, vpt);
    } else if constexpr (MODE == rope3d::kModeFusedSP) {
        // head-scatter stores: adjacent pairing and same-dtype caches only
        if (pairing != ROPE3D_PAIRING_ADJACENT || cache_fmt != rope3d::kCacheSame) return nullptr;
        return dtype == ROPE3D_BF16
                   ? pick_trig<__nv_bfloat16, MODE, rope3d::kPairAdjacent, rope3d::kCacheSame>(trig, vpt)
                   : pick_trig<float, MODE, rope3d::kPairAdjacent, rope3d::kCacheSame>(trig, vpt);
    } else if constexpr (MODE == rope3d::kModeApply) {
        return dtype == ROPE3D_BF16
                   ? pick_pairing<__nv_bfloat16, MODE, rope3d::kCacheSame>(pairing, trig, vpt)
                   : pick_pairing<float, MODE, rope3d::kCacheSame>(pairing, trig, vpt);
    } else {
        return dtype == ROPE3D_BF16 ? pick_format<__nv_bfloat16, MODE>(cache_fmt, pairing, trig, vpt)
                                    : pick_format<float, MODE>(cache_fmt, pairing, trig, vpt);
    }
}

using TmaKernelFn = void (*)(const rope3d::Params);

template <typename T, int TRIG, int PAIR, bool CFP8>
TmaKernelFn pick_tma_vpt(int vpt) {
    if constexpr (PAIR == rope3d::kPairHalf) {
        switch (vpt) {
            case 2: return rope3d::qk_norm_rope_tma_kernel<T, 2, TRIG, PAIR, CFP8>;
            case 4: return rope3d::qk_norm_rope_tma_kernel<T, 4, TRIG, PAIR, CFP8>;
#if ROPE3D_MAX_VPT >= 6
            case 6: return rope3d::qk_norm_rope_tma_kernel<T, 6, TRIG, PAIR, CFP8>;
#endif
            default: return nullptr;
        }
    } else {
        switch (vpt) {
            case 1: return rope3d::qk_norm_rope_tma_kernel<T, 1, TRIG, PAIR, CFP8>;
            case 2: return rope3d::qk_norm_rope_tma_kernel<T, 2, TRIG, PAIR, CFP8>;
            case 3: return rope3d::qk_norm_rope_tma_kernel<T, 3, TRIG, PAIR, CFP8>;
            case 4: return rope3d::qk_norm_rope_tma_kernel<T, 4, TRIG, PAIR, CFP8>;
#if ROPE3D_MAX_VPT >= 6
            case 5: return rope3d::qk_norm_rope_tma_kernel<T, 5, TRIG, PAIR, CFP8>;
            case 6: return rope3d::qk_norm_rope_tma_kernel<T, 6, TRIG, PAIR, CFP8>;
#endif
            default: return nullptr;
        }
    }
}

template <typename T, int PAIR, bool CFP8>
TmaKernelFn pick_tma_trig(int trig, int vpt) {
    return trig == ROPE3D_TRIG_TABLE ? pick_tma_vpt<T, rope3d::kTrigTable, PAIR, CFP8>(vpt)
                                     : pick_tma_vpt<T, rope3d::kTrigOnTheFly, PAIR, CFP8>(vpt);
}

template <typename T, bool CFP8>
TmaKernelFn pick_tma_pairing(int pairing, int trig, int vpt) {
    return pairing == ROPE3D_PAIRING_HALF ? pick_tma_trig<T, rope3d::kPairHalf, CFP8>(trig, vpt)
                                          : pick_tma_trig<T, rope3d::kPairAdjacent, CFP8>(trig, vpt);
}

TmaKernelFn pick_tma_kernel(int dtype, int trig, int pairing, bool fp8, int vpt) {
    if (dtype == ROPE3D_BF16)
        return fp8 ? pick_tma_pairing<__nv_bfloat16, true>(pairing, trig, vpt)
                   : pick_tma_pairing<__nv_bfloat16, false>(pairing, trig, vpt);
    return fp8 ? pick_tma_pairing<float, true>(pairing, trig, vpt)
               : pick_tma_pairing<float, false>(pairing, trig, vpt);
}

// Resident blocks per SM for a kernel at a block size and shared-memory size.  The
// first use of a kernel on a device raises its dynamic shared-memory limit to the
// device's opt-in maximum (a per-kernel setting, so it is set once and never lowered).
// Both are cached per device.
struct OccKey {
    int dev;
    KernelFn fn;
    int threads;
    size_t smem;
    int blocks;
};
std::vector<OccKey> g_occ;
std::vector<std::pair<int, KernelFn>> g_smem_raised;

int occupancy(int dev, KernelFn fn, int threads, size_t smem, int max_smem, int* blocks) {
    bool raised = false;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        for (const OccKey& k : g_occ)
            if (k.dev == dev && k.fn == fn && k.threads == threads && k.smem == smem) {
                *blocks = k.blocks;
                return ROPE3D_OK;
            }
        for (const auto& r : g_smem_raised)
            if (r.first == dev && r.second == fn) raised = true;
    }
    cudaError_t e;
    if (!raised) {
        e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
        if (e != cudaSuccess)
            return fail(ROPE3D_ECUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        std::lock_guard<std::mutex> lock(g_mutex);
        g_smem_raised.emplace_back(dev, fn);
    }
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, reinterpret_cast<const void*>(fn),
                                                      threads, smem);
    if (e != cudaSuccess)
        return fail(ROPE3D_ECUDA, "cudaOccupancyMaxActiveBlocksPerMultiprocessor: %s",
                    cudaGetErrorString(e));
    if (n < 1) return fail(ROPE3D_EINVAL, "a block of %d threads with %zu bytes of shared "
                                          "memory does not fit on an SM", threads, smem);
    std::lock_guard<std::mutex> lock(g_mutex);
    g_occ.push_back(OccKey{dev, fn, threads, smem, n});
    *blocks = n;
    return ROPE3D_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch with programmatic stream serialisation: the kernel may start while the
// previous kernel on the stream drains, and waits for it (griddepcontrol.wait) before
// it touches global memory.
cudaError_t launch_pdl(const void* fn, int64_t grid, int threads, size_t smem,
                       cudaStream_t stream, rope3d::Params* p) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {p};
    return cudaLaunchKernelExC(&cfg, fn, args);
}

// Shared-memory plan of the TMA kernel for `teams` teams of `stages` stages each;
// returns the total dynamic shared memory and fills the offsets.
size_t tma_layout(rope3d::Params& p, int teams, int stages, int warps_per_team) {
    size_t off = 0;
    p.off_bars = (uint32_t)off;
    off += (size_t)teams * stages * sizeof(uint64_t);
    off = align_up(off, 16);
    p.off_fail = (uint32_t)off;
    off += (size_t)teams * sizeof(int);
    off = align_up(off, 16);
    p.off_part = (uint32_t)off;
    off += (size_t)2 * teams * warps_per_team * sizeof(float2);
    off = align_up(off, 16);
    p.off_w = (uint32_t)off;
    off += (size_t)2 * p.dim * sizeof(float);
    off = align_up(off, 128);
    p.off_stage = (uint32_t)off;
    off += (size_t)teams * stages * 3 * p.row_bytes;
    return off;
}

#ifndef ROPE3D_TMA_MAX_STAGES
#define ROPE3D_TMA_MAX_STAGES 3
#endif

// The fused step through the bulk-copy ring, when a ring of at least two stages per
// team fits in shared memory; *launched stays false if it launched nothing (the caller
// falls back to the register kernel).  Unless `forced`, the ring is also declined where
// the register kernel measured faster on B200 (graph-replayed launches, 2 to 64 heads,
// 1560 to 32760 tokens): teams under 96 threads, a single team per block, or fewer
// than 16 rows per team.  The ring won by 2-5% at 24 to 40 heads and >= 10800 tokens.
int launch_fused_tma(rope3d::Params& p, int64_t N, int dtype, int trig, int pairing, int dev,
                     const DeviceInfo& info, cudaStream_t stream, bool forced, bool* launched) {
    *launched = false;
    if (p.k_bscale != nullptr) return ROPE3D_OK;  // NVFP4 caches: register kernel only
    const Geometry g = geometry(N, dtype, pairing);
    if (g.tpr > rope3d::kTmaMaxBlockThreads || g.vpt > ROPE3D_MAX_VPT) return ROPE3D_OK;
    const int warps_per_team = g.tpr / 32;
    p.row_bytes = (uint32_t)(N * rope3d::kHeadDim * (dtype == ROPE3D_BF16 ? 2 : 4));
    int teams = (ROPE3D_TMA_BLOCK_TARGET < rope3d::kTmaMaxBlockThreads
                     ? ROPE3D_TMA_BLOCK_TARGET : rope3d::kTmaMaxBlockThreads) / g.tpr;
    if (teams < 1) teams = 1;
    if (teams > rope3d::kMaxTeamsPerBlock) teams = rope3d::kMaxTeamsPerBlock;
    if ((int64_t)teams > p.units) teams = (int)p.units;
    int stages = 0;
    size_t smem = 0;
    for (; teams >= 1; --teams) {
        for (stages = ROPE3D_TMA_MAX_STAGES; stages >= 2; --stages) {
            smem = tma_layout(p, teams, stages, warps_per_team);
            if (smem <= (size_t)info.max_smem_optin) break;
        }
        if (stages >= 2) break;
    }
    if (teams < 1 || stages < 2) return ROPE3D_OK;  // does not fit: register kernel
    // Measured on B200: the ring pays off for wide rows and long runs only, and not with an
    // FP8 cache in adjacent pairing, where the register kernel's extra resident warps hide
    // the quantizer's latency better (127 vs 139 us on the 720P chunk).
    if (!forced && (g.tpr < 96 || teams < 2 ||
                    p.units < (int64_t)16 * info.sms * teams ||
                    (p.k_scale != nullptr && pairing == ROPE3D_PAIRING_ADJACENT)))
        return ROPE3D_OK;
    smem = tma_layout(p, teams, stages, warps_per_team);
    TmaKernelFn fn = pick_tma_kernel(dtype, trig, pairing, p.k_scale != nullptr, g.vpt);
    if (fn == nullptr) return ROPE3D_OK;
    const int threads = teams * g.tpr;
    int per_sm = 0;
    int rc = occupancy(dev, fn, threads, smem, info.max_smem_optin, &per_sm);
    if (rc != ROPE3D_OK) return rc;
    const int64_t needed = (p.units + teams - 1) / teams;
    int64_t grid = (int64_t)info.sms * per_sm;
    if (grid > needed) grid = needed;
    p.dim_vecs = g.dim_vecs;
    p.tpr = g.tpr;
    p.teams = teams;
    p.stages = stages;
    p.wait_limit_ns = g_wait_limit_ns.load();
    p.tx_extra = g_tx_extra.load();
    const cudaError_t e =
        launch_pdl(reinterpret_cast<const void*>(fn), grid, threads, smem, stream, &p);
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "kernel launch: %s", cudaGetErrorString(e));
    *launched = true;
    return ok();
}

template <int MODE>
int launch(rope3d::Params& p, int64_t N, int dtype, int trig, int pairing, int dev,
           const DeviceInfo& info, cudaStream_t stream) {
    const Geometry g = geometry(N, dtype, pairing);
    const int max_threads = g.vpt > 4 ? rope3d::kMaxBlockThreads / 2 : rope3d::kMaxBlockThreads;
    if (g.tpr > max_threads || g.vpt > ROPE3D_MAX_VPT)
        return fail(ROPE3D_EINVAL, "N=%lld heads is more than one row team can hold",
                    (long long)N);
    int teams = (ROPE3D_REG_BLOCK_TARGET < max_threads ? ROPE3D_REG_BLOCK_TARGET
                                                       : max_threads) / g.tpr;
    if (teams < 1) teams = 1;
    if (teams > rope3d::kMaxTeamsPerBlock) teams = rope3d::kMaxTeamsPerBlock;
    if ((int64_t)teams > p.units) teams = (int)p.units;
    const int threads = teams * g.tpr;
    const int warps_per_team = g.tpr / 32;
    size_t smem = 0;
    if (MODE != rope3d::kModeApply) {
        smem = (size_t)2 * p.dim * sizeof(float);
        if (warps_per_team > 1) smem += (size_t)2 * teams * warps_per_team * sizeof(float2);
        if (MODE == rope3d::kModeFusedSP) smem += 3 * rope3d::kMaxRanks * sizeof(void*);
        if (p.k_bscale != nullptr) smem += rope3d::kNvfp4TableFloats * sizeof(float);
    }
    if (smem > (size_t)info.max_smem_optin)
        return fail(ROPE3D_EINVAL, "N=%lld needs %zu bytes of shared memory (limit %d)",
                    (long long)N, smem, info.max_smem_optin);
    const int cache_fmt = p.k_bscale != nullptr ? rope3d::kCacheNvfp4
                          : p.k_scale != nullptr ? rope3d::kCacheFp8 : rope3d::kCacheSame;
    KernelFn fn = pick_kernel<MODE>(dtype, trig, pairing, cache_fmt, g.vpt);
    if (fn == nullptr) return fail(ROPE3D_EINVAL, "no kernel for vpt=%d", g.vpt);
    int per_sm = 0;
    int rc = occupancy(dev, fn, threads, smem, info.max_smem_optin, &per_sm);
    if (rc != ROPE3D_OK) return rc;
    const int64_t needed = (p.units + teams - 1) / teams;
    int64_t grid = (int64_t)info.sms * per_sm;
    if (grid > needed) grid = needed;
    p.dim_vecs = g.dim_vecs;
    p.tpr = g.tpr;
    p.teams = teams;
    const cudaError_t e =
        launch_pdl(reinterpret_cast<const void*>(fn), grid, threads, smem, stream, &p);
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "kernel launch: %s", cudaGetErrorString(e));
    return ok();
}

// ---------------------------------------------------------------- QKV projection (tcgen05)

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2-D tensor map of a row-major bf16 matrix [rows][cols] read in boxes of box_rows x 64
// with the 128-byte swizzle; rows past the end read as zero.
int make_map_bf16(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr) return fail(ROPE3D_ECUDA, "cuTensorMapEncodeTiled is not available");
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)rope3d::kGemmBK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ROPE3D_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return ROPE3D_OK;
}

int launch_qkv_gemm(const void* x, const void* w, rope3d::GemmParams& gp, int dev,
                    const DeviceInfo& info, cudaStream_t stream) {
    // the pair form (two CTAs of a cluster per 256x256 tile, each loading half of W's rows;
    // measured 6% faster at 720P) or cta_group::1 (one CTA per 128x256 tile)
    const int G = g_gemm_cta_group.load() == 2 ? 2 : 1;
    CUtensorMap map_x, map_w;
    int rc = make_map_bf16(&map_x, x, gp.M, gp.K, rope3d::kGemmBM);
    if (rc != ROPE3D_OK) return rc;
    rc = make_map_bf16(&map_w, w, gp.n_out, gp.K, rope3d::kGemmBN / G);
    if (rc != ROPE3D_OK) return rc;
    gp.num_m = (gp.M + rope3d::kGemmBM * G - 1) / (rope3d::kGemmBM * G);
    gp.num_n = (gp.n_out + rope3d::kGemmBN - 1) / rope3d::kGemmBN;
    gp.wait_limit_ns = g_wait_limit_ns.load();
    gp.tx_extra = g_tx_extra.load();
    const void* fn = G == 2 ? reinterpret_cast<const void*>(rope3d::qkv_proj_kernel<2>)
                            : reinterpret_cast<const void*>(rope3d::qkv_proj_kernel<1>);
    if ((int)rope3d::kGemmSmemBytes > info.max_smem_optin)
        return fail(ROPE3D_EDEVICE, "the projection needs %zu bytes of shared memory",
                    rope3d::kGemmSmemBytes);
    static std::once_flag raised[2][64];
    cudaError_t e = cudaSuccess;
    std::call_once(raised[G - 1][dev & 63], [&] {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)rope3d::kGemmSmemBytes);
    });
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    const int tiles = gp.num_m * gp.num_n;
    const int slots = info.sms / G;  // one CTA per SM (shared memory, tensor memory)
    const int grid = G * (tiles < slots ? tiles : slots);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(rope3d::kGemmThreads);
    cfg.dynamicSmemBytes = rope3d::kGemmSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&map_x, &map_w, &gp};
    e = cudaLaunchKernelExC(&cfg, fn, args);
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "projection launch: %s", cudaGetErrorString(e));
    return ROPE3D_OK;
}

void fill_common(rope3d::Params& p, int64_t B, int64_t N, int64_t token_begin, int64_t token_end,
                 int64_t frame_offset, int H, int W, const rope3d_tables* tables) {
    p.n_tok = token_end - token_begin;
    p.units = B * p.n_tok;
    p.token_begin = token_begin;
    p.frame_offset = frame_offset;
    p.hw = (int64_t)H * W;
    p.H = H;
    p.W = W;
    p.dim = (int)(N * rope3d::kHeadDim);
    p.inv_dim = 1.0f / (float)p.dim;
    p.n_t = tables->n_t;
    p.n_h = tables->n_h;
    p.n_w = tables->n_w;
    p.tab_t = tables->tab_t;
    p.tab_h = tables->tab_h;
    p.tab_w = tables->tab_w;
    p.tab_rows_t = tables->max_t;
    p.tab_rows_h = tables->max_h;
    p.tab_rows_w = tables->max_w;
    p.check_shrink = g_check_shrink.load();
    std::memcpy(p.inv_freq, tables->inv_freq, sizeof(p.inv_freq));
    p.status = tables->d_status;
    p.cache_tokens = 1;  // the fused entry point overwrites these two
    p.slot = 0;
}

void set_small_idx(rope3d::Params& p) {
    const int64_t lim = (int64_t)1 << 31;
    p.small_idx = (p.units < lim && p.token_begin + p.n_tok + p.slot < lim &&
                   p.cache_tokens < lim && p.hw < lim) ? 1 : 0;
    if (p.small_idx) {
        p.div_ntok = rope3d::make_fastdiv((uint32_t)p.n_tok);
        p.div_hw = rope3d::make_fastdiv((uint32_t)p.hw);
        p.div_w = rope3d::make_fastdiv((uint32_t)p.W);
        p.div_cache = rope3d::make_fastdiv((uint32_t)p.cache_tokens);
    }
}

// The options of a call (NULL = all defaults), checked.
int read_options(const rope3d_options* options, rope3d_options* out, bool with_cache) {
    rope3d_options o{};
    if (options != nullptr) o = *options;
    if (o.pairing != ROPE3D_PAIRING_ADJACENT && o.pairing != ROPE3D_PAIRING_HALF)
        return fail(ROPE3D_EINVAL, "options.pairing %d is not a ROPE3D_PAIRING_* value",
                    o.pairing);
    if (o.cache_layout != ROPE3D_CACHE_TOKEN_MAJOR && o.cache_layout != ROPE3D_CACHE_HEAD_MAJOR)
        return fail(ROPE3D_EINVAL, "options.cache_layout %d is not a ROPE3D_CACHE_* value",
                    o.cache_layout);
    if (!with_cache && o.cache_layout != ROPE3D_CACHE_TOKEN_MAJOR)
        return fail(ROPE3D_EINVAL, "options.cache_layout applies to the fused step only");
    if (o.cache_dtype != ROPE3D_CACHE_SAME && o.cache_dtype != ROPE3D_CACHE_FP8_E4M3 &&
        o.cache_dtype != ROPE3D_CACHE_NVFP4)
        return fail(ROPE3D_EINVAL, "options.cache_dtype %d is not a ROPE3D_CACHE_* value",
                    o.cache_dtype);
    if (!with_cache && (o.cache_dtype != ROPE3D_CACHE_SAME || o.k_scale || o.v_scale))
        return fail(ROPE3D_EINVAL, "options.cache_dtype and scales apply to the fused step only");
    if (o.cache_dtype == ROPE3D_CACHE_FP8_E4M3 || o.cache_dtype == ROPE3D_CACHE_NVFP4) {
        if (o.k_scale == nullptr || o.v_scale == nullptr)
            return fail(ROPE3D_EINVAL, "a quantized cache needs k_scale and v_scale");
        const uintptr_t mask = o.cache_dtype == ROPE3D_CACHE_FP8_E4M3 ? 3u : 7u;
        if ((reinterpret_cast<uintptr_t>(o.k_scale) & mask) ||
            (reinterpret_cast<uintptr_t>(o.v_scale) & mask))
            return fail(ROPE3D_EALIGN, "k_scale and v_scale must be %d-byte aligned",
                        (int)mask + 1);
    } else if (o.k_scale != nullptr || o.v_scale != nullptr) {
        return fail(ROPE3D_EINVAL, "k_scale / v_scale are only for a quantized cache");
    }
    if (o.cache_dtype == ROPE3D_CACHE_NVFP4) {
        for (float g : {o.nvfp4_k_global, o.nvfp4_v_global})
            if (!(g >= 0.0f) || !std::isfinite(g))
                return fail(ROPE3D_EINVAL, "NVFP4 global scales must be finite and >= 0 (0 = 1)");
        if (o.nvfp4_k_global == 0.0f) o.nvfp4_k_global = 1.0f;
        if (o.nvfp4_v_global == 0.0f) o.nvfp4_v_global = 1.0f;
    } else if (o.nvfp4_k_global != 0.0f || o.nvfp4_v_global != 0.0f) {
        return fail(ROPE3D_EINVAL, "NVFP4 global scales are only for an NVFP4 cache");
    }
    if (o.reserved0 != 0) return fail(ROPE3D_EINVAL, "options.reserved0 must be zero");
    for (int r : o.reserved)
        if (r != 0) return fail(ROPE3D_EINVAL, "options.reserved must be zero");
    *out = o;
    return ROPE3D_OK;
}

void fill_layout(rope3d::Params& p, int64_t N, int dtype, const rope3d_options& o) {
    const int vph = rope3d::kHeadDim / (dtype == ROPE3D_BF16 ? 8 : 4);
    p.cache_head_major = o.cache_layout == ROPE3D_CACHE_HEAD_MAJOR ? 1 : 0;
    p.n_heads = (int)N;
    p.vph_log2 = vph == 16 ? 4 : 5;
    p.k_scale = o.cache_dtype == ROPE3D_CACHE_FP8_E4M3 ? o.k_scale : nullptr;
    p.v_scale = o.cache_dtype == ROPE3D_CACHE_FP8_E4M3 ? o.v_scale : nullptr;
    const bool fp4 = o.cache_dtype == ROPE3D_CACHE_NVFP4;
    p.k_bscale = fp4 ? reinterpret_cast<uint8_t*>(o.k_scale) : nullptr;
    p.v_bscale = fp4 ? reinterpret_cast<uint8_t*>(o.v_scale) : nullptr;
    p.k_global = fp4 ? o.nvfp4_k_global : 1.0f;
    p.v_global = fp4 ? o.nvfp4_v_global : 1.0f;
    // k = fp32(1 / fp32(6 g)), as the format's rounding recipe defines it
    const float six_k = 6.0f * p.k_global, six_v = 6.0f * p.v_global;
    p.k_inv6g = 1.0f / six_k;
    p.v_inv6g = 1.0f / six_v;
}

int check_tables_device(const rope3d_tables* tables, int dev) {
    if (tables->device != dev)
        return fail(ROPE3D_EDEVICE, "tables were built on device %d, current device is %d",
                    tables->device, dev);
    return ROPE3D_OK;
}

}  // namespace

extern "C" {

int rope3d_version(void) { return 10000; }

const char* rope3d_strerror(int status) {
    switch (status) {
        case ROPE3D_OK: return "success";
        case ROPE3D_EINVAL: return "invalid argument";
        case ROPE3D_ERANGE: return "index range out of bounds";
        case ROPE3D_ECUDA: return "CUDA runtime error";
        case ROPE3D_EDEVICE: return "unsupported or mismatched device";
        case ROPE3D_EALIGN: return "tensor pointer not 16-byte aligned";
        case ROPE3D_EOVERLAP: return "output buffers overlap";
        case ROPE3D_ETIMEOUT: return "a kernel wait timed out";
        case ROPE3D_EINDEX: return "a device-side index check failed (checked build)";
        default: return "unknown status";
    }
}

const char* rope3d_last_error(void) { return g_last_error; }

int rope3d_tables_init(rope3d_tables** out, int head_dim, int n_t, int n_h, int n_w,
                       double theta, int max_t, int max_h, int max_w, int schedule,
                       void* cuda_stream) {
    if (out == nullptr) return fail(ROPE3D_EINVAL, "out is NULL");
    *out = nullptr;
    if (n_t < 0 || n_h < 0 || n_w < 0 || head_dim != 2 * (n_t + n_h + n_w))
        return fail(ROPE3D_EINVAL, "head_dim %d != 2 (n_t + n_h + n_w) = 2 (%d + %d + %d)",
                    head_dim, n_t, n_h, n_w);
    if (head_dim != rope3d::kHeadDim)
        return fail(ROPE3D_EINVAL, "head_dim %d: the kernels support %d", head_dim,
                    rope3d::kHeadDim);
    if (!(theta > 1.0) || !std::isfinite(theta))
        return fail(ROPE3D_EINVAL, "theta must be finite and > 1");
    if (schedule != ROPE3D_SCHEDULE_PER_AXIS && schedule != ROPE3D_SCHEDULE_HEAD_WIDE)
        return fail(ROPE3D_EINVAL, "schedule %d is not a ROPE3D_SCHEDULE_* value", schedule);
    if (max_t < 0 || max_h < 0 || max_w < 0)
        return fail(ROPE3D_EINVAL, "table sizes must be >= 0");
    const bool with_tables = max_t > 0 || max_h > 0 || max_w > 0;
    if (with_tables && (max_t == 0 || max_h == 0 || max_w == 0))
        return fail(ROPE3D_EINVAL, "max_t, max_h, max_w must be all zero or all positive");
    if ((int64_t)max_t * n_t + (int64_t)max_h * n_h + (int64_t)max_w * n_w > (int64_t)1 << 28)
        return fail(ROPE3D_EINVAL, "tables too large");
    DeviceInfo info;
    int dev = 0;
    int rc = device_info(&info, &dev);
    if (rc != ROPE3D_OK) return rc;

    rope3d_tables* tb = new rope3d_tables();
    tb->device = dev;
    tb->head_dim = head_dim;
    tb->n_t = n_t;
    tb->n_h = n_h;
    tb->n_w = n_w;
    tb->theta = theta;
    tb->schedule = schedule;
    tb->max_t = max_t;
    tb->max_h = max_h;
    tb->max_w = max_w;
    tb->d_tab = nullptr;
    tb->d_status = nullptr;
    {
        cudaError_t e = cudaMalloc(&tb->d_status, 16);
        if (e == cudaSuccess) e = cudaMemset(tb->d_status, 0, 16);
        if (e != cudaSuccess) {
            if (tb->d_status) cudaFree(tb->d_status);
            delete tb;
            return fail(ROPE3D_ECUDA, "status word allocation: %s", cudaGetErrorString(e));
        }
    }

    // Inverse frequency of every pair, in double, then the fp32 copy the on-the-fly
    // path multiplies positions by.
    const int n_axis[3] = {n_t, n_h, n_w};
    const int pairs = n_t + n_h + n_w;
    double inv[rope3d::kPairs];
    int first = 0;
    for (int a = 0; a < 3; ++a) {
        for (int j = 0; j < n_axis[a]; ++j) {
            const double e = schedule == ROPE3D_SCHEDULE_PER_AXIS
                                 ? (double)(2 * j) / (double)(2 * n_axis[a])
                                 : (double)(2 * (first + j)) / (double)(2 * pairs);
            inv[first + j] = std::pow(theta, -e);
            tb->inv_freq[first + j] = (float)inv[first + j];
        }
        first += n_axis[a];
    }

    if (with_tables) {
        const int max_pos[3] = {max_t, max_h, max_w};
        size_t count = 0;
        for (int a = 0; a < 3; ++a) count += (size_t)max_pos[a] * n_axis[a];
        std::vector<float2> host(count);
        size_t off = 0;
        size_t axis_off[3];
        first = 0;
        for (int a = 0; a < 3; ++a) {
            axis_off[a] = off;
            for (int p = 0; p < max_pos[a]; ++p)
                for (int j = 0; j < n_axis[a]; ++j) {
                    const double phi = (double)p * inv[first + j];
                    host[off++] = make_float2((float)std::cos(phi), (float)std::sin(phi));
                }
            first += n_axis[a];
        }
        cudaError_t e = cudaMalloc(&tb->d_tab, count * sizeof(float2));
        if (e != cudaSuccess) {
            cudaFree(tb->d_status);
            delete tb;
            return fail(ROPE3D_ECUDA, "cudaMalloc(%zu): %s", count * sizeof(float2),
                        cudaGetErrorString(e));
        }
        cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
        e = cudaMemcpyAsync(tb->d_tab, host.data(), count * sizeof(float2),
                            cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
        if (e != cudaSuccess) {
            cudaFree(tb->d_tab);
            cudaFree(tb->d_status);
            delete tb;
            return fail(ROPE3D_ECUDA, "table upload: %s", cudaGetErrorString(e));
        }
        tb->tab_t = tb->d_tab + axis_off[0];
        tb->tab_h = tb->d_tab + axis_off[1];
        tb->tab_w = tb->d_tab + axis_off[2];
    } else {
        tb->tab_t = tb->tab_h = tb->tab_w = nullptr;
    }
    *out = tb;
    return ok();
}

void rope3d_tables_destroy(rope3d_tables* tables) {
    if (tables == nullptr) return;
    int cur = 0;
    cudaGetDevice(&cur);
    if (cur != tables->device) cudaSetDevice(tables->device);
    cudaDeviceSynchronize();
    if (tables->d_tab != nullptr) cudaFree(tables->d_tab);
    if (tables->d_status != nullptr) cudaFree(tables->d_status);
    if (cur != tables->device) cudaSetDevice(cur);
    delete tables;
}

namespace {

// Reads the device status word at d_status in stream order, clears it when set, and maps
// it to a status code.
int read_status_word(int* d_status, cudaStream_t stream) {
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, d_status, sizeof(int), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && word != 0) e = cudaMemsetAsync(d_status, 0, sizeof(int), stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "status read: %s", cudaGetErrorString(e));
    if (word & rope3d::kStatusWaitTimeout)
        return fail(ROPE3D_ETIMEOUT, "a kernel gave up waiting for a shared-memory stage to fill");
    if (word & rope3d::kStatusIndexRange)
        return fail(ROPE3D_EINDEX, "a kernel of the checked build derived a cache, table or "
                                   "destination row outside its extent and skipped it");
    return ok();
}

}  // namespace

int rope3d_check_device_status(const rope3d_tables* tables, void* cuda_stream) {
    if (tables == nullptr) return fail(ROPE3D_EINVAL, "tables is NULL");
    int cur = 0;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (cur != tables->device)
        return fail(ROPE3D_EDEVICE, "tables were built on device %d, current device is %d",
                    tables->device, cur);
    return read_status_word(tables->d_status, static_cast<cudaStream_t>(cuda_stream));
}

void rope3d_testing_set_waits(uint64_t wait_limit_ns, uint32_t tx_extra_bytes) {
    g_wait_limit_ns.store(wait_limit_ns ? wait_limit_ns : kDefaultWaitLimitNs);
    g_tx_extra.store(tx_extra_bytes);
}

int rope3d_testing_last_path(void) { return g_last_path; }

uint32_t rope3d_testing_fast_divide(uint32_t n, uint32_t d) {
    if (d == 0 || d >= (1u << 31) || n >= (1u << 31)) return 0xFFFFFFFFu;
    return rope3d::fast_div(n, rope3d::make_fastdiv(d));
}

int rope3d_testing_shrink_checked_cache(int64_t shrink_rows) {
    if (shrink_rows < 0) return fail(ROPE3D_EINVAL, "shrink_rows %lld < 0", (long long)shrink_rows);
    g_check_shrink.store(shrink_rows);
    return ok();
}

int rope3d_testing_gemm_cta_group(int group) {
    if (group != 0 && group != 1 && group != 2)
        return fail(ROPE3D_EINVAL, "group %d is not 0, 1 or 2", group);
    g_gemm_cta_group.store(group == 0 ? 2 : group);
    return ok();
}

int rope3d_testing_force_path(int path) {
    if (path != ROPE3D_PATH_AUTO && path != ROPE3D_PATH_REGISTERS && path != ROPE3D_PATH_TMA)
        return fail(ROPE3D_EINVAL, "path %d is not a ROPE3D_PATH_* value", path);
    g_force_path.store(path);
    return ok();
}

int rope3d_qk_norm_rope_append(const void* q, const void* k, const void* v, void* q_out,
                               int64_t B, int64_t N, int D, int dtype,
                               int64_t token_begin, int64_t token_end, int64_t frame_offset,
                               int T, int H, int W,
                               const float* q_norm_w, const float* k_norm_w, float eps,
                               void* k_cache, void* v_cache, int64_t cache_tokens,
                               int64_t slot, const rope3d_tables* tables, int trig,
                               void* cuda_stream) {
    return rope3d_qk_norm_rope_append_ex(q, k, v, q_out, B, N, D, dtype, token_begin, token_end,
                                         frame_offset, T, H, W, q_norm_w, k_norm_w, eps, k_cache,
                                         v_cache, cache_tokens, slot, tables, trig, nullptr,
                                         cuda_stream);
}

int rope3d_qk_norm_rope_append_ex(const void* q, const void* k, const void* v, void* q_out,
                                  int64_t B, int64_t N, int D, int dtype,
                                  int64_t token_begin, int64_t token_end, int64_t frame_offset,
                                  int T, int H, int W,
                                  const float* q_norm_w, const float* k_norm_w, float eps,
                                  void* k_cache, void* v_cache, int64_t cache_tokens,
                                  int64_t slot, const rope3d_tables* tables, int trig,
                                  const rope3d_options* options, void* cuda_stream) {
    rope3d_options opt;
    int rc = read_options(options, &opt, true);
    if (rc != ROPE3D_OK) return rc;
    rc = check_common(B, N, D, dtype, token_begin, token_end, frame_offset, T, H, W, tables,
                          trig);
    if (rc != ROPE3D_OK) return rc;
    if (!q || !k || !v || !q_out || !k_cache || !v_cache || !q_norm_w || !k_norm_w)
        return fail(ROPE3D_EINVAL, "a tensor pointer is NULL");
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return fail(ROPE3D_EINVAL, "eps must be >= 0");
    if (cache_tokens < 1) return fail(ROPE3D_EINVAL, "cache_tokens must be >= 1");
    if (slot < 0) return fail(ROPE3D_EINVAL, "slot must be >= 0");
    if (token_end - token_begin > cache_tokens)
        return fail(ROPE3D_ERANGE, "%lld tokens do not fit a cache of %lld rows",
                    (long long)(token_end - token_begin), (long long)cache_tokens);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_out) ||
        !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q_norm_w) ||
        !aligned16(k_norm_w))
        return fail(ROPE3D_EALIGN, "every tensor pointer must be 16-byte aligned");
    const size_t esz = dtype == ROPE3D_BF16 ? 2 : 4;
    const size_t row = (size_t)N * D * esz;
    const size_t act = (size_t)B * (size_t)(token_end - token_begin) * row;
    const bool fp8 = opt.cache_dtype == ROPE3D_CACHE_FP8_E4M3;
    const bool fp4 = opt.cache_dtype == ROPE3D_CACHE_NVFP4;
    const size_t heads = (size_t)B * (size_t)cache_tokens * (size_t)N;
    const size_t cache = fp4 ? heads * D / 2 : fp8 ? heads * D : heads * D * esz;
    if (fp8 || fp4) {
        const size_t sc = heads * (fp8 ? sizeof(float) : (size_t)D / 16);
        const void* bufs[6] = {q, k, v, q_out, k_cache, v_cache};
        const size_t sizes[6] = {act, act, act, act, cache, cache};
        for (int b2 = 0; b2 < 6; ++b2)
            if (overlap(opt.k_scale, sc, bufs[b2], sizes[b2]) ||
                overlap(opt.v_scale, sc, bufs[b2], sizes[b2]))
                return fail(ROPE3D_EOVERLAP, "a scale array overlaps a tensor");
        if (overlap(opt.k_scale, sc, opt.v_scale, sc))
            return fail(ROPE3D_EOVERLAP, "k_scale overlaps v_scale");
    }
    if (q_out != q && overlap(q_out, act, q, act))
        return fail(ROPE3D_EOVERLAP, "q_out partly overlaps q (only exact in-place is allowed)");
    if (overlap(q_out, act, k, act) || overlap(q_out, act, v, act) ||
        overlap(q_out, act, k_cache, cache) || overlap(q_out, act, v_cache, cache))
        return fail(ROPE3D_EOVERLAP, "q_out overlaps k, v or a cache");
    if (overlap(k_cache, cache, v_cache, cache) || overlap(k_cache, cache, q, act) ||
        overlap(k_cache, cache, k, act) || overlap(k_cache, cache, v, act) ||
        overlap(v_cache, cache, q, act) || overlap(v_cache, cache, k, act) ||
        overlap(v_cache, cache, v, act))
        return fail(ROPE3D_EOVERLAP, "a cache overlaps the other cache or an input");

    DeviceInfo info;
    int dev = 0;
    rc = device_info(&info, &dev);
    if (rc != ROPE3D_OK) return rc;
    rc = check_tables_device(tables, dev);
    if (rc != ROPE3D_OK) return rc;

    rope3d::Params p{};
    fill_common(p, B, N, token_begin, token_end, frame_offset, H, W, tables);
    p.q = q;
    p.k = k;
    p.v = v;
    p.q_out = q_out;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.q_w = q_norm_w;
    p.k_w = k_norm_w;
    p.cache_tokens = cache_tokens;
    p.slot = slot;
    p.eps = eps;
    fill_layout(p, N, dtype, opt);
    set_small_idx(p);
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    const int path = g_force_path.load();
    if (path != ROPE3D_PATH_REGISTERS) {
        bool launched = false;
        rc = launch_fused_tma(p, N, dtype, trig, opt.pairing, dev, info, stream,
                              path == ROPE3D_PATH_TMA, &launched);
        if (launched) g_last_path = ROPE3D_PATH_TMA;
        if (rc != ROPE3D_OK || launched) return rc;
        if (path == ROPE3D_PATH_TMA)
            return fail(ROPE3D_EINVAL, "the TMA path does not take this call (N=%lld%s)",
                        (long long)N, p.k_bscale ? ", NVFP4 cache" : "");
    }
    rc = launch<rope3d::kModeFused>(p, N, dtype, trig, opt.pairing, dev, info, stream);
    if (rc == ROPE3D_OK) g_last_path = ROPE3D_PATH_REGISTERS;
    return rc;
}

int rope3d_qk_norm_rope_append_sp(const void* q, const void* k, const void* v,
                                  int64_t B, int64_t N, int D, int dtype,
                                  int64_t token_begin, int64_t token_end, int64_t frame_offset,
                                  int T, int H, int W,
                                  const float* q_norm_w, const float* k_norm_w, float eps,
                                  const rope3d_sp_dest* dest, int64_t cache_tokens,
                                  int64_t slot, const rope3d_tables* tables, int trig,
                                  const rope3d_options* options, void* cuda_stream) {
    rope3d_options opt;
    int rc = read_options(options, &opt, true);
    if (rc != ROPE3D_OK) return rc;
    rc = check_common(B, N, D, dtype, token_begin, token_end, frame_offset, T, H, W, tables,
                      trig);
    if (rc != ROPE3D_OK) return rc;
    if (opt.pairing != ROPE3D_PAIRING_ADJACENT || opt.cache_dtype != ROPE3D_CACHE_SAME)
        return fail(ROPE3D_EINVAL,
                    "head-scatter stores support adjacent pairing and same-dtype caches");
    if (!q || !k || !v || !q_norm_w || !k_norm_w || !dest)
        return fail(ROPE3D_EINVAL, "a tensor pointer or dest is NULL");
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return fail(ROPE3D_EINVAL, "eps must be >= 0");
    const int P = dest->ranks;
    if (P < 1 || P > ROPE3D_SP_MAX_RANKS)
        return fail(ROPE3D_EINVAL, "dest->ranks %d is not in [1, %d]", P, ROPE3D_SP_MAX_RANKS);
    if (N % P != 0)
        return fail(ROPE3D_EINVAL, "N=%lld heads do not split evenly over %d ranks",
                    (long long)N, P);
    if (dest->reserved0 != 0) return fail(ROPE3D_EINVAL, "dest->reserved0 must be zero");
    if (cache_tokens < 1) return fail(ROPE3D_EINVAL, "cache_tokens must be >= 1");
    if (slot < 0) return fail(ROPE3D_EINVAL, "slot must be >= 0");
    if (token_end - token_begin > cache_tokens)
        return fail(ROPE3D_ERANGE, "%lld tokens do not fit a cache of %lld rows",
                    (long long)(token_end - token_begin), (long long)cache_tokens);
    if (dest->q_row0 < 0 || dest->q_rows < 1 || token_begin < dest->q_row0 ||
        token_end > dest->q_row0 + dest->q_rows)
        return fail(ROPE3D_ERANGE, "tokens [%lld, %lld) are not inside the q rows [%lld, %lld)",
                    (long long)token_begin, (long long)token_end, (long long)dest->q_row0,
                    (long long)(dest->q_row0 + dest->q_rows));
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_norm_w) ||
        !aligned16(k_norm_w))
        return fail(ROPE3D_EALIGN, "every tensor pointer must be 16-byte aligned");
    for (int r = 0; r < P; ++r) {
        if (!dest->q[r] || !dest->k_cache[r] || !dest->v_cache[r])
            return fail(ROPE3D_EINVAL, "a destination pointer of rank %d is NULL", r);
        if (!aligned16(dest->q[r]) || !aligned16(dest->k_cache[r]) ||
            !aligned16(dest->v_cache[r]))
            return fail(ROPE3D_EALIGN, "destination pointers must be 16-byte aligned");
    }
    // Overlap among the local inputs and the destinations is checked for destinations in
    // this process's address space only as far as the ranges are known here: inputs must
    // not overlap any destination range of a rank.
    const size_t esz = dtype == ROPE3D_BF16 ? 2 : 4;
    const size_t act = (size_t)B * (size_t)(token_end - token_begin) * (size_t)N * D * esz;
    const size_t qd = (size_t)B * (size_t)dest->q_rows * (size_t)(N / P) * D * esz;
    const size_t cd = (size_t)B * (size_t)cache_tokens * (size_t)(N / P) * D * esz;
    for (int r = 0; r < P; ++r) {
        const void* dsts[3] = {dest->q[r], dest->k_cache[r], dest->v_cache[r]};
        const size_t dsz[3] = {qd, cd, cd};
        for (int j = 0; j < 3; ++j)
            if (overlap(dsts[j], dsz[j], q, act) || overlap(dsts[j], dsz[j], k, act) ||
                overlap(dsts[j], dsz[j], v, act))
                return fail(ROPE3D_EOVERLAP, "a destination of rank %d overlaps an input", r);
        for (int r2 = 0; r2 < P; ++r2) {
            const void* d2[3] = {dest->q[r2], dest->k_cache[r2], dest->v_cache[r2]};
            for (int j = 0; j < 3; ++j)
                for (int j2 = 0; j2 < 3; ++j2)
                    if ((r2 != r || j2 != j) && overlap(dsts[j], dsz[j], d2[j2], dsz[j2]))
                        return fail(ROPE3D_EOVERLAP, "destination buffers overlap");
        }
    }

    DeviceInfo info;
    int dev = 0;
    rc = device_info(&info, &dev);
    if (rc != ROPE3D_OK) return rc;
    rc = check_tables_device(tables, dev);
    if (rc != ROPE3D_OK) return rc;

    rope3d::Params p{};
    fill_common(p, B, N, token_begin, token_end, frame_offset, H, W, tables);
    p.q = q;
    p.k = k;
    p.v = v;
    p.q_w = q_norm_w;
    p.k_w = k_norm_w;
    p.cache_tokens = cache_tokens;
    p.slot = slot;
    p.eps = eps;
    fill_layout(p, N, dtype, opt);
    p.sp_ranks = P;
    p.sp_heads = (int)(N / P);
    p.sp_q_rows = dest->q_rows;
    p.sp_q_row0 = dest->q_row0;
    for (int r = 0; r < P; ++r) {
        p.sp_dst[3 * r] = dest->q[r];
        p.sp_dst[3 * r + 1] = dest->k_cache[r];
        p.sp_dst[3 * r + 2] = dest->v_cache[r];
    }
    set_small_idx(p);
    rc = launch<rope3d::kModeFusedSP>(p, N, dtype, trig, opt.pairing, dev, info,
                                      static_cast<cudaStream_t>(cuda_stream));
    if (rc == ROPE3D_OK) g_last_path = ROPE3D_PATH_REGISTERS;
    return rc;
}

namespace {

int check_projection(const void* x, const void* w_qkv, const float* b_qkv, int64_t M, int64_t K,
                     int64_t N, int D) {
    if (!x || !w_qkv) return fail(ROPE3D_EINVAL, "x or w_qkv is NULL");
    if (D != rope3d::kHeadDim) return fail(ROPE3D_EINVAL, "head size D=%d must be 128", D);
    if (N < 1 || M < 1) return fail(ROPE3D_EINVAL, "N=%lld and M=%lld must be >= 1",
                                    (long long)N, (long long)M);
    if (K < rope3d::kGemmBK || K % rope3d::kGemmBK != 0 || K > (1 << 20))
        return fail(ROPE3D_EINVAL, "input features K=%lld must be a multiple of %d",
                    (long long)K, rope3d::kGemmBK);
    if (M > (1 << 30) || 3 * N * D > (1 << 24))
        return fail(ROPE3D_ERANGE, "M=%lld or N=%lld is too large", (long long)M, (long long)N);
    // the kernels count output tiles (128 x 256 at the smallest) in an int
    const int64_t tiles = ((M + rope3d::kGemmBM - 1) / rope3d::kGemmBM) *
                          ((3 * N * D + rope3d::kGemmBN - 1) / rope3d::kGemmBN);
    if (tiles >= ((int64_t)1 << 31))
        return fail(ROPE3D_ERANGE, "M=%lld x 3 N D=%lld is %lld output tiles, over 2^31 - 1",
                    (long long)M, (long long)(3 * N * D), (long long)tiles);
    if (!aligned16(x) || !aligned16(w_qkv) ||
        (b_qkv != nullptr && (reinterpret_cast<uintptr_t>(b_qkv) & 3u)))
        return fail(ROPE3D_EALIGN, "x and w_qkv must be 16-byte aligned, b_qkv 4-byte");
    return ROPE3D_OK;
}

}  // namespace

int rope3d_qkv_project(const void* x, const void* w_qkv, const float* b_qkv, int64_t M,
                       int64_t K, int64_t N, int D, void* q_out, void* k_out, void* v_out,
                       void* cuda_stream) {
    int rc = check_projection(x, w_qkv, b_qkv, M, K, N, D);
    if (rc != ROPE3D_OK) return rc;
    if (!q_out || !k_out || !v_out) return fail(ROPE3D_EINVAL, "an output pointer is NULL");
    if (!aligned16(q_out) || !aligned16(k_out) || !aligned16(v_out))
        return fail(ROPE3D_EALIGN, "outputs must be 16-byte aligned");
    const size_t out = (size_t)M * N * D * 2;
    const size_t xb = (size_t)M * K * 2, wb = (size_t)3 * N * D * K * 2;
    const void* outs[3] = {q_out, k_out, v_out};
    for (int a = 0; a < 3; ++a) {
        if (overlap(outs[a], out, x, xb) || overlap(outs[a], out, w_qkv, wb))
            return fail(ROPE3D_EOVERLAP, "an output overlaps x or w_qkv");
        for (int b = a + 1; b < 3; ++b)
            if (overlap(outs[a], out, outs[b], out)) return fail(ROPE3D_EOVERLAP, "outputs overlap");
    }
    DeviceInfo info;
    int dev = 0;
    rc = device_info(&info, &dev);
    if (rc != ROPE3D_OK) return rc;
    rope3d::GemmParams gp{};
    gp.M = (int)M;
    gp.K = (int)K;
    gp.dim = (int)(N * D);
    gp.n_out = 3 * gp.dim;
    gp.bias = b_qkv;
    gp.q_out = static_cast<__nv_bfloat16*>(q_out);
    gp.k_out = static_cast<__nv_bfloat16*>(k_out);
    gp.v_cache = static_cast<__nv_bfloat16*>(v_out);  // a cache of M rows, row = token
    gp.n_tok = M;
    gp.token_begin = 0;
    gp.cache_tokens = M;
    gp.slot = 0;
    gp.n_heads = (int)N;
    gp.cache_head_major = 0;
    gp.status = nullptr;
    return launch_qkv_gemm(x, w_qkv, gp, dev, info, static_cast<cudaStream_t>(cuda_stream));
}

size_t rope3d_qkv_workspace_bytes(int64_t B, int64_t n_tok, int64_t N, int D) {
    if (B < 1 || n_tok < 1 || N < 1 || D != rope3d::kHeadDim) return 0;
    const int64_t M = B * n_tok, dim = N * D;
    if (dim % rope3d::kGemmBN == 0)  // fused epilogue: partial sums of squares per row and tile
        return (size_t)(2 * M * (dim / rope3d::kGemmBN)) * sizeof(float);
    return (size_t)(M * dim) * 2;  // odd head counts: k is staged for the step
}

int rope3d_qkv_norm_rope_append(const void* x, const void* w_qkv, const float* b_qkv, int64_t K,
                                int64_t B, int64_t N, int D, int64_t token_begin,
                                int64_t token_end, int64_t frame_offset, int T, int H, int W,
                                const float* q_norm_w, const float* k_norm_w, float eps,
                                void* q_out, void* workspace, size_t workspace_bytes,
                                void* k_cache, void* v_cache, int64_t cache_tokens, int64_t slot,
                                const rope3d_tables* tables, int trig,
                                const rope3d_options* options, void* cuda_stream) {
    void* k_work = workspace;
    rope3d_options opt;
    int rc = read_options(options, &opt, true);
    if (rc != ROPE3D_OK) return rc;
    if (opt.pairing != ROPE3D_PAIRING_ADJACENT || opt.cache_dtype != ROPE3D_CACHE_SAME)
        return fail(ROPE3D_EINVAL, "the projection-fed step supports adjacent pairing and "
                                   "bf16 caches");
    rc = check_common(B, N, D, ROPE3D_BF16, token_begin, token_end, frame_offset, T, H, W,
                      tables, trig);
    if (rc != ROPE3D_OK) return rc;
    const int64_t n_tok = token_end - token_begin;
    rc = check_projection(x, w_qkv, b_qkv, B * n_tok, K, N, D);
    if (rc != ROPE3D_OK) return rc;
    if (!q_out || !k_work || !k_cache || !v_cache || !q_norm_w || !k_norm_w)
        return fail(ROPE3D_EINVAL, "a tensor pointer is NULL");
    const size_t ws_need = rope3d_qkv_workspace_bytes(B, n_tok, N, D);
    if (workspace_bytes < ws_need)
        return fail(ROPE3D_EINVAL, "workspace of %zu bytes, %zu needed", workspace_bytes, ws_need);
    const bool fused = (N * D) % rope3d::kGemmBN == 0;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return fail(ROPE3D_EINVAL, "eps must be >= 0");
    if (cache_tokens < 1) return fail(ROPE3D_EINVAL, "cache_tokens must be >= 1");
    if (slot < 0) return fail(ROPE3D_EINVAL, "slot must be >= 0");
    if (n_tok > cache_tokens)
        return fail(ROPE3D_ERANGE, "%lld tokens do not fit a cache of %lld rows",
                    (long long)n_tok, (long long)cache_tokens);
    if (!aligned16(q_out) || !aligned16(k_work) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(q_norm_w) || !aligned16(k_norm_w))
        return fail(ROPE3D_EALIGN, "every tensor pointer must be 16-byte aligned");
    const size_t act = (size_t)B * n_tok * N * D * 2;
    const size_t cache = (size_t)B * cache_tokens * N * D * 2;
    const size_t xb = (size_t)B * n_tok * K * 2, wb = (size_t)3 * N * D * K * 2;
    const void* bufs[4] = {q_out, k_work, k_cache, v_cache};
    const size_t sizes[4] = {act, ws_need, cache, cache};
    for (int a = 0; a < 4; ++a) {
        if (overlap(bufs[a], sizes[a], x, xb) || overlap(bufs[a], sizes[a], w_qkv, wb))
            return fail(ROPE3D_EOVERLAP, "an output overlaps x or w_qkv");
        for (int b = a + 1; b < 4; ++b)
            if (overlap(bufs[a], sizes[a], bufs[b], sizes[b]))
                return fail(ROPE3D_EOVERLAP, "q_out, the workspace and the caches must not overlap");
    }
    DeviceInfo info;
    int dev = 0;
    rc = device_info(&info, &dev);
    if (rc != ROPE3D_OK) return rc;
    rc = check_tables_device(tables, dev);
    if (rc != ROPE3D_OK) return rc;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);

    // 1. q, k, v = QKV(x): q into q_out, k into k_work, v into the V cache rows
    rope3d::GemmParams gp{};
    gp.M = (int)(B * n_tok);
    gp.K = (int)K;
    gp.dim = (int)(N * D);
    gp.n_out = 3 * gp.dim;
    gp.bias = b_qkv;
    gp.q_out = static_cast<__nv_bfloat16*>(q_out);
    gp.k_out = static_cast<__nv_bfloat16*>(k_work);
    gp.v_cache = static_cast<__nv_bfloat16*>(v_cache);
    gp.n_tok = n_tok;
    gp.token_begin = token_begin;
    gp.cache_tokens = cache_tokens;
    gp.slot = slot;
    gp.n_heads = (int)N;
    gp.cache_head_major = opt.cache_layout == ROPE3D_CACHE_HEAD_MAJOR ? 1 : 0;
    gp.status = tables->d_status;
    if (fused) {
        // 1+2. the projection with the normalisation and rotation in its epilogue
        const int64_t M = B * n_tok;
        gp.fused = 1;
        gp.q_w = q_norm_w;
        gp.k_w = k_norm_w;
        gp.eps = eps;
        gp.inv_dim = 1.0f / (float)(N * D);
        gp.k_cache = static_cast<__nv_bfloat16*>(k_cache);
        gp.psum = static_cast<float*>(workspace);
        const bool table = trig == ROPE3D_TRIG_TABLE;
        gp.tab_t = table ? tables->tab_t : nullptr;
        gp.tab_h = table ? tables->tab_h : nullptr;
        gp.tab_w = table ? tables->tab_w : nullptr;
        gp.n_t = tables->n_t;
        gp.n_h = tables->n_h;
        gp.n_w = tables->n_w;
        gp.H = H;
        gp.W = W;
        gp.hw = (int64_t)H * W;
        gp.frame_offset = frame_offset;
        for (int j = 0; j < rope3d::kPairs; ++j) gp.inv_freq[j] = tables->inv_freq[j];
        rc = launch_qkv_gemm(x, w_qkv, gp, dev, info, stream);
        if (rc != ROPE3D_OK) return rc;
        // 3. the per-row scale 1 / sqrt(mean + eps) of q and K, in place
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)((2 * M + rope3d::kScaleWarps - 1) / rope3d::kScaleWarps));
        cfg.blockDim = dim3(32 * rope3d::kScaleWarps);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        void* args[] = {&gp};
        const cudaError_t e = cudaLaunchKernelExC(
            &cfg, reinterpret_cast<const void*>(rope3d::qk_row_scale_kernel), args);
        if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "row scale launch: %s", cudaGetErrorString(e));
        g_last_path = ROPE3D_PATH_REGISTERS;
        return ROPE3D_OK;
    }
    rc = launch_qkv_gemm(x, w_qkv, gp, dev, info, stream);
    if (rc != ROPE3D_OK) return rc;

    // 2. the step on q (in place) and k; V is already in the cache
    rope3d::Params p{};
    fill_common(p, B, N, token_begin, token_end, frame_offset, H, W, tables);
    p.q = q_out;
    p.k = k_work;
    p.v = nullptr;
    p.q_out = q_out;
    p.k_cache = k_cache;
    p.v_cache = nullptr;
    p.q_w = q_norm_w;
    p.k_w = k_norm_w;
    p.cache_tokens = cache_tokens;
    p.slot = slot;
    p.eps = eps;
    fill_layout(p, N, ROPE3D_BF16, opt);
    set_small_idx(p);
    rc = launch<rope3d::kModeFusedNoV>(p, N, ROPE3D_BF16, trig, opt.pairing, dev, info, stream);
    if (rc == ROPE3D_OK) g_last_path = ROPE3D_PATH_REGISTERS;
    return rc;
}

int rope3d_sp_output_all_to_all(const void* o, int64_t B, int64_t L, int64_t heads_per_rank,
                                int D, int dtype, const rope3d_sp_out_dest* dest,
                                void* cuda_stream) {
    if (o == nullptr || dest == nullptr) return fail(ROPE3D_EINVAL, "o or dest is NULL");
    if (D != rope3d::kHeadDim) return fail(ROPE3D_EINVAL, "head size D=%d, not %d", D,
                                           rope3d::kHeadDim);
    if (dtype != ROPE3D_F32 && dtype != ROPE3D_BF16)
        return fail(ROPE3D_EINVAL, "dtype %d is neither ROPE3D_F32 nor ROPE3D_BF16", dtype);
    if (B < 1 || L < 1 || heads_per_rank < 1)
        return fail(ROPE3D_EINVAL, "B=%lld, L=%lld and heads_per_rank=%lld must be >= 1",
                    (long long)B, (long long)L, (long long)heads_per_rank);
    const int P = dest->ranks;
    if (P < 1 || P > ROPE3D_SP_MAX_RANKS)
        return fail(ROPE3D_EINVAL, "dest->ranks %d is not in [1, %d]", P, ROPE3D_SP_MAX_RANKS);
    if (dest->rank < 0 || dest->rank >= P)
        return fail(ROPE3D_EINVAL, "dest->rank %d is not in [0, %d)", dest->rank, P);
    if (dest->cuts[0] != 0 || dest->cuts[P] != L)
        return fail(ROPE3D_ERANGE, "cuts must run from 0 to L = %lld", (long long)L);
    for (int r = 0; r < P; ++r)
        if (dest->cuts[r + 1] < dest->cuts[r])
            return fail(ROPE3D_ERANGE, "cuts must not fall (cuts[%d] > cuts[%d])", r, r + 1);
    if (!aligned16(o)) return fail(ROPE3D_EALIGN, "o must be 16-byte aligned");
    const size_t esz = dtype == ROPE3D_BF16 ? 2 : 4;
    const size_t row = (size_t)heads_per_rank * D * esz;
    const size_t o_bytes = (size_t)B * (size_t)L * row;
    size_t out_bytes[ROPE3D_SP_MAX_RANKS];
    for (int r = 0; r < P; ++r) {
        out_bytes[r] = (size_t)B * (size_t)(dest->cuts[r + 1] - dest->cuts[r]) * row * P;
        if (out_bytes[r] == 0) continue;
        if (dest->out[r] == nullptr)
            return fail(ROPE3D_EINVAL, "dest->out[%d] is NULL but its slice is not empty", r);
        if (!aligned16(dest->out[r]))
            return fail(ROPE3D_EALIGN, "dest->out[%d] must be 16-byte aligned", r);
        if (overlap(dest->out[r], out_bytes[r], o, o_bytes))
            return fail(ROPE3D_EOVERLAP, "dest->out[%d] overlaps o", r);
        for (int r2 = 0; r2 < r; ++r2)
            if (out_bytes[r2] && overlap(dest->out[r], out_bytes[r], dest->out[r2], out_bytes[r2]))
                return fail(ROPE3D_EOVERLAP, "dest->out[%d] overlaps dest->out[%d]", r, r2);
    }
    DeviceInfo info;
    int dev = 0;
    int rc = device_info(&info, &dev);
    if (rc != ROPE3D_OK) return rc;

    // 32-byte units when o, every destination and the row length allow them
    bool wide = ROPE3D_A2A_WIDE && row % 32 == 0 && aligned32(o);
    for (int r = 0; r < P; ++r)
        if (out_bytes[r] && !aligned32(dest->out[r])) wide = false;
    const int unit = wide ? 32 : 16;
    rope3d::SpOutParams sp{};
    sp.o = static_cast<const unsigned char*>(o);
    for (int r = 0; r < P; ++r) sp.out[r] = static_cast<unsigned char*>(dest->out[r]);
    for (int r = 0; r <= P; ++r) sp.cuts[r] = dest->cuts[r];
    for (int r = P + 1; r <= rope3d::kMaxRanks; ++r) sp.cuts[r] = L;
    sp.L = L;
    sp.ranks = P;
    sp.rank = dest->rank;
    sp.row_units = (int)(row / unit);
    sp.out_row_units = sp.row_units * P;
    sp.total = B * L * sp.row_units;
    sp.small = sp.total < ((int64_t)1 << 31) ? 1 : 0;
    if (sp.small) {
        sp.div_row = rope3d::make_fastdiv((uint32_t)sp.row_units);
        sp.div_L = rope3d::make_fastdiv((uint32_t)L);
    }
    constexpr int U = ROPE3D_A2A_UNROLL;
    const int threads = 256;
    int64_t grid = (sp.total + (int64_t)threads * U - 1) / ((int64_t)threads * U);
    const int64_t cap = (int64_t)info.sms * 8;
    if (grid > cap) grid = cap;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(threads);
    cfg.stream = static_cast<cudaStream_t>(cuda_stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&sp};
    const void* fn = wide ? reinterpret_cast<const void*>(rope3d::sp_output_all_to_all_kernel<32, U>)
                          : reinterpret_cast<const void*>(rope3d::sp_output_all_to_all_kernel<16, U>);
    const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "kernel launch: %s", cudaGetErrorString(e));
    return ok();
}

int rope3d_apply(const void* x, void* out, int64_t B, int64_t N, int D, int dtype,
                 int64_t token_begin, int64_t token_end, int64_t frame_offset,
                 int T, int H, int W, const rope3d_tables* tables, int trig,
                 void* cuda_stream) {
    return rope3d_apply_ex(x, out, B, N, D, dtype, token_begin, token_end, frame_offset, T, H,
                           W, tables, trig, nullptr, cuda_stream);
}

int rope3d_apply_ex(const void* x, void* out, int64_t B, int64_t N, int D, int dtype,
                    int64_t token_begin, int64_t token_end, int64_t frame_offset,
                    int T, int H, int W, const rope3d_tables* tables, int trig,
                    const rope3d_options* options, void* cuda_stream) {
    rope3d_options opt;
    int rc = read_options(options, &opt, false);
    if (rc != ROPE3D_OK) return rc;
    rc = check_common(B, N, D, dtype, token_begin, token_end, frame_offset, T, H, W, tables,
                          trig);
    if (rc != ROPE3D_OK) return rc;
    if (!x || !out) return fail(ROPE3D_EINVAL, "a tensor pointer is NULL");
    if (!aligned16(x) || !aligned16(out))
        return fail(ROPE3D_EALIGN, "every tensor pointer must be 16-byte aligned");
    const size_t esz = dtype == ROPE3D_BF16 ? 2 : 4;
    const size_t act = (size_t)B * (size_t)(token_end - token_begin) * (size_t)N * D * esz;
    if (out != x && overlap(out, act, x, act))
        return fail(ROPE3D_EOVERLAP, "out partly overlaps x (only exact in-place is allowed)");
    DeviceInfo info;
    int dev = 0;
    rc = device_info(&info, &dev);
    if (rc != ROPE3D_OK) return rc;
    rc = check_tables_device(tables, dev);
    if (rc != ROPE3D_OK) return rc;
    rope3d::Params p{};
    fill_common(p, B, N, token_begin, token_end, frame_offset, H, W, tables);
    p.q = x;
    p.q_out = out;
    fill_layout(p, N, dtype, opt);
    set_small_idx(p);
    return launch<rope3d::kModeApply>(p, N, dtype, trig, opt.pairing, dev, info,
                                      static_cast<cudaStream_t>(cuda_stream));
}

int rope3d_decode_positions(int64_t token_begin, int64_t token_end, int64_t frame_offset,
                            int T, int H, int W, int64_t cache_tokens, int64_t slot,
                            int64_t* out, void* cuda_stream) {
    if (T < 1 || H < 1 || W < 1)
        return fail(ROPE3D_EINVAL, "grid T=%d H=%d W=%d must be >= 1", T, H, W);
    if (frame_offset < 0 || cache_tokens < 1 || slot < 0)
        return fail(ROPE3D_EINVAL, "frame_offset, slot must be >= 0 and cache_tokens >= 1");
    if (token_begin < 0 || token_end <= token_begin)
        return fail(ROPE3D_ERANGE, "token range [%lld, %lld) is empty or negative",
                    (long long)token_begin, (long long)token_end);
    if (token_end > (int64_t)T * H * W)
        return fail(ROPE3D_ERANGE, "token_end exceeds T*H*W");
    if (out == nullptr) return fail(ROPE3D_EINVAL, "out is NULL");
    if ((reinterpret_cast<uintptr_t>(out) & 7u) != 0)
        return fail(ROPE3D_EALIGN, "out must be 8-byte aligned");
    DeviceInfo info;
    int dev = 0;
    int rc = device_info(&info, &dev);
    if (rc != ROPE3D_OK) return rc;
    const int64_t n = token_end - token_begin;
    const int threads = 256;
    const int64_t blocks = (n + threads - 1) / threads;
    int64_t hw = (int64_t)H * W;
    void* args[] = {&token_begin, const_cast<int64_t*>(&n), &frame_offset, &hw, &W, &H,
                    &cache_tokens, &slot, &out};
    const cudaError_t e = cudaLaunchKernel(
        reinterpret_cast<const void*>(&rope3d::decode_positions_kernel), dim3((unsigned)blocks),
        dim3(threads), args, 0, static_cast<cudaStream_t>(cuda_stream));
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "kernel launch: %s", cudaGetErrorString(e));
    return ok();
}

}  // extern "C"

// ---------------------------------------------------------------- no-allocation entry point
//
// rope3d_qk_norm_rope_append_noalloc serves callers that cannot call cudaMalloc (see
// include/rope3d.h).  Everything the fused step needs beyond the caller's inputs and
// outputs -- the cos/sin rows of this call's positions and the status word of the
// bounded waits -- lives in one file-scope device array instead of a rope3d_tables
// allocation.  The array exists on every GPU that loads this library until the process
// exits.  Every call shares it and it keeps the last call's contents; each call writes
// its own table rows and clears the status word first.  Calls that overlap on the GPU
// (different streams, or different host threads) race on it.

namespace {

constexpr int kNoAllocStatusBytes = 256;       // status word, padded to the array's alignment
constexpr int kNoAllocTableEntries = 8192;     // (cos, sin) pairs: 64 KiB
constexpr size_t kNoAllocScratchBytes = kNoAllocStatusBytes + kNoAllocTableEntries * sizeof(float2);

std::mutex g_noalloc_mutex;
std::vector<void*> g_noalloc_addr;            // per device: device address of the array
float2 g_noalloc_host[kNoAllocTableEntries];  // host staging of one call's rows (under the mutex)

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of the array on the current device.  Host code sees only a host-side
// stand-in under the array's name, so the real address is asked for once per device,
// with that device current, and remembered.
int noalloc_scratch_address(int dev, unsigned char** out) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if ((int)g_noalloc_addr.size() <= dev) g_noalloc_addr.resize(dev + 1, nullptr);
    if (g_noalloc_addr[dev] == nullptr) {
        void* ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr)
            return fail(ROPE3D_ECUDA, "cudaGetSymbolAddress of the scratch array: %s",
                        cudaGetErrorString(e));
        g_noalloc_addr[dev] = ptr;
    }
    *out = static_cast<unsigned char*>(g_noalloc_addr[dev]);
    return ROPE3D_OK;
}

}  // namespace

extern "C" int rope3d_qk_norm_rope_append_noalloc(
    const void* q, const void* k, const void* v, void* q_out, int64_t B, int64_t N, int D,
    int dtype, int64_t token_begin, int64_t token_end, int64_t frame_offset, int T, int H, int W,
    const float* q_norm_w, const float* k_norm_w, float eps, void* k_cache, void* v_cache,
    int64_t cache_tokens, int64_t slot, int n_t, int n_h, int n_w, double theta, int schedule,
    int trig, void* cuda_stream) {
    if (n_t < 0 || n_h < 0 || n_w < 0 || 2 * (n_t + n_h + n_w) != rope3d::kHeadDim)
        return fail(ROPE3D_EINVAL, "n_t + n_h + n_w must be %d", rope3d::kHeadDim / 2);
    if (!(theta > 1.0) || !std::isfinite(theta))
        return fail(ROPE3D_EINVAL, "theta must be finite and > 1");
    if (schedule != ROPE3D_SCHEDULE_PER_AXIS && schedule != ROPE3D_SCHEDULE_HEAD_WIDE)
        return fail(ROPE3D_EINVAL, "schedule %d is not a ROPE3D_SCHEDULE_* value", schedule);
    if (trig != ROPE3D_TRIG_TABLE && trig != ROPE3D_TRIG_ONTHEFLY)
        return fail(ROPE3D_EINVAL, "trig %d is not a ROPE3D_TRIG_* value", trig);
    if (T < 1 || H < 1 || W < 1 || frame_offset < 0 || token_begin < 0 ||
        token_end <= token_begin || token_end > (int64_t)T * H * W)
        return fail(ROPE3D_ERANGE, "grid or token range invalid");

    // Rows of the three tables this call reads: frames [t_first, t_last], all H rows and
    // all W columns.  They must fit the array.
    const int64_t hw = (int64_t)H * W;
    const int64_t t_first = frame_offset + token_begin / hw;
    const int64_t t_last = frame_offset + (token_end - 1) / hw;
    const int64_t entries = (t_last - t_first + 1) * n_t + (int64_t)H * n_h + (int64_t)W * n_w;
    if (trig == ROPE3D_TRIG_TABLE && entries > kNoAllocTableEntries)
        return fail(ROPE3D_ERANGE,
                    "this call needs %lld cos/sin entries; the no-allocation scratch holds %d "
                    "(use ROPE3D_TRIG_ONTHEFLY or the rope3d_tables entry points)",
                    (long long)entries, kNoAllocTableEntries);

    DeviceInfo info;
    int dev = 0;
    int rc = device_info(&info, &dev);
    if (rc != ROPE3D_OK) return rc;
    unsigned char* scratch = nullptr;
    rc = noalloc_scratch_address(dev, &scratch);
    if (rc != ROPE3D_OK) return rc;

    // A frequency configuration on the stack that points into the scratch array.
    rope3d_tables tb{};
    tb.device = dev;
    tb.head_dim = rope3d::kHeadDim;
    tb.n_t = n_t;
    tb.n_h = n_h;
    tb.n_w = n_w;
    tb.theta = theta;
    tb.schedule = schedule;
    tb.d_status = reinterpret_cast<int*>(scratch);
    const int n_axis[3] = {n_t, n_h, n_w};
    const int pairs = n_t + n_h + n_w;
    double inv[rope3d::kPairs];
    int first = 0;
    for (int a = 0; a < 3; ++a) {
        for (int j = 0; j < n_axis[a]; ++j) {
            const double e = schedule == ROPE3D_SCHEDULE_PER_AXIS
                                 ? (double)(2 * j) / (double)(2 * n_axis[a])
                                 : (double)(2 * (first + j)) / (double)(2 * pairs);
            inv[first + j] = std::pow(theta, -e);
            tb.inv_freq[first + j] = (float)inv[first + j];
        }
        first += n_axis[a];
    }
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(int), stream);
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "status clear: %s", cudaGetErrorString(e));
    if (trig == ROPE3D_TRIG_TABLE) {
        // fp64 cos/sin of position * inv_freq stored as fp32, as rope3d_tables_init does
        float2* h = g_noalloc_host;
        size_t off = 0;
        for (int64_t p = t_first; p <= t_last; ++p)
            for (int j = 0; j < n_t; ++j) {
                const double phi = (double)p * inv[j];
                h[off++] = make_float2((float)std::cos(phi), (float)std::sin(phi));
            }
        const size_t off_h = off;
        for (int p = 0; p < H; ++p)
            for (int j = 0; j < n_h; ++j) {
                const double phi = (double)p * inv[n_t + j];
                h[off++] = make_float2((float)std::cos(phi), (float)std::sin(phi));
            }
        const size_t off_w = off;
        for (int p = 0; p < W; ++p)
            for (int j = 0; j < n_w; ++j) {
                const double phi = (double)p * inv[n_t + n_h + j];
                h[off++] = make_float2((float)std::cos(phi), (float)std::sin(phi));
            }
        float2* d_tab = reinterpret_cast<float2*>(scratch + kNoAllocStatusBytes);
        // A copy from pageable memory has taken the host rows (staged or copied) when it
        // returns, so the next call may refill g_noalloc_host once it holds the lock; the
        // device array is written in stream order, ahead of this call's kernel.
        e = cudaMemcpyAsync(d_tab, h, off * sizeof(float2), cudaMemcpyHostToDevice, stream);
        if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "table upload: %s", cudaGetErrorString(e));
        tb.d_tab = d_tab;
        // the t rows start at frame t_first; the kernel indexes them by global frame
        tb.tab_t = reinterpret_cast<float2*>(reinterpret_cast<uintptr_t>(d_tab) -
                                             (uintptr_t)(t_first * n_t) * sizeof(float2));
        tb.tab_h = d_tab + off_h;
        tb.tab_w = d_tab + off_w;
        tb.max_t = (int)(t_last + 1);
        tb.max_h = H;
        tb.max_w = W;
    }
    return rope3d_qk_norm_rope_append(q, k, v, q_out, B, N, D, dtype, token_begin, token_end,
                                      frame_offset, T, H, W, q_norm_w, k_norm_w, eps, k_cache,
                                      v_cache, cache_tokens, slot, &tb, trig, cuda_stream);
}

extern "C" int rope3d_noalloc_check_status(void* cuda_stream) {
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(ROPE3D_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    unsigned char* scratch = nullptr;
    const int rc = noalloc_scratch_address(dev, &scratch);
    if (rc != ROPE3D_OK) return rc;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    return read_status_word(reinterpret_cast<int*>(scratch),
                            static_cast<cudaStream_t>(cuda_stream));
}
