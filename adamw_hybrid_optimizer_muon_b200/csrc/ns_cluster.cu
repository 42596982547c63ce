// The whole Newton-Schulz chain of a short unit in one launch, held in the
// shared memory of a thread-block cluster.
//
// For units with at most 128 rows (m <= 128: per-head slices of Q/K/V, small
// matrices; "Qwen Training Details...", "Confirmed": per-head
// orthogonalisation) the tile kernel spends most of each iteration moving X:
// the Gram is a single 128 x 128 tile with a long K loop, and the apply
// reads X and the Gram again. Here a cluster of kCl CTAs owns one unit for
// all N iterations ("MuonClip Optimizer", "Newton-Schulz Orthogonalization":
// X <- aX + b (X X^T) X, the short-side form of X <- 1.5X - 0.5 X(X^T X)):
//
//   * CTA r keeps columns [r*NC, (r+1)*NC) of X (NC <= 512, bf16) in shared
//     memory for the whole chain, loaded once by TMA;
//   * Gram: each CTA forms its partial A_r = X_r X_r^T (128 x 128, fp32 in
//     TMEM) with tcgen05, then the cluster reduce-scatters: CTA r sends rows
//     [16d, 16d + 16) of A_r to CTA d's receive buffer (distributed shared
//     memory); CTA d adds its 16 rows over the eight sources in a fixed
//     order, scales by b (times s^2 on the first iteration, s = 1/(||u||+eps)),
//     rounds to bf16 and writes them into every CTA's copy of B;
//   * apply: X_r' = s*(a X_r + B X_r) with tcgen05 (B from shared memory, X_r
//     as the MN-major operand), written back over X_r in shared memory;
//   * the last iteration writes W <- W*(1 - lr*wd) - lr*scale*X_N into the
//     caller's fp32 weights; X_N is never rounded.
//
// Only the first load of X and the final read-modify-write of W touch HBM.
// Every sum has a fixed order, so results do not depend on scheduling.
// Waits are bounded; after a timeout a CTA skips its work but takes part in
// every cluster barrier, then drains its MMAs and its load before it exits.
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace ma {

namespace {

constexpr int kCl = 8;                           // CTAs per cluster (one unit)
constexpr int kRows = 128;                       // rows of a unit, padded (M of every MMA)
constexpr int kMaxNC = 512;                      // columns of X per CTA
constexpr int kThreads = 256;                    // 8 warps: two per TMEM lane quadrant
constexpr uint32_t kPanel = kRows * 128;         // one 64-column panel of X or B: 128 rows x 128 B
constexpr uint32_t kXBytes = kMaxNC / 64 * kPanel;       // 128 KB
constexpr uint32_t kBBytes = 2 * kPanel;                 // 32 KB: B, 128 x 128 bf16, two K panels
constexpr int kSlabRows = kRows / kCl;                   // 16 rows of A reduced by each CTA
constexpr uint32_t kSlab = kSlabRows * kRows * 4;        // 8 KB: one source's rows for one reducer
constexpr uint32_t kRxBytes = kCl * kSlab;               // 64 KB
constexpr uint32_t kTmemCols = 512;
constexpr long long kDrainNs = 50000000LL;

struct ClCtl {
    uint64_t load;  // X block landed
    uint64_t mma;   // one commit per MMA batch (Gram, apply)
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t commits;  // MMA batches committed so far
    int32_t waited;   // of those, the ones whose completion thread 0 has seen
};

constexpr size_t kSmem = 1024 + kXBytes + kBBytes + kRxBytes + 256;
static_assert(kSmem <= 232448, "shared memory");
static_assert(sizeof(ClCtl) <= 256, "control block");

// Byte offset of element (row, col) of a 128-row panel set with the 128-byte
// swizzle (16-byte chunk index XOR row % 8), bf16 elements.
__device__ __forceinline__ uint32_t panel_off(int row, int col) {
    const uint32_t chunk = (uint32_t)((col & 63) >> 3) ^ (uint32_t)(row & 7);
    return (uint32_t)(col >> 6) * kPanel + (uint32_t)row * 128u + (chunk << 4) + (uint32_t)(col & 7) * 2u;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void fence_proxy_async_cluster() {
    asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}

__device__ __forceinline__ float update_w(float w, float x, float decay, float lrs, float lr_wd, int cautious) {
    if (cautious) return (x * w > 0.f ? w - lr_wd * w : w) - lrs * x;
    return w * decay - lrs * x;
}

__global__ void __cluster_dims__(kCl, 1, 1) __launch_bounds__(kThreads, 1)
    ns_cluster_kernel(const __grid_constant__ NsClusterLaunch L) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Xs = smem;                  // this CTA's columns of X, 64-column panels
    uint8_t* Bs = Xs + kXBytes;          // B = b*A (bf16), two 64-column K panels
    uint8_t* Rx = Bs + kBBytes;          // fp32 [source][16 rows][128 columns], this CTA's rows of A
    ClCtl* ctl = reinterpret_cast<ClCtl*>(Rx + kRxBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t r = cluster_ctarank();
    const int u = (int)cluster_id_x();  // one unit per cluster
    const int m = L.m, n = L.n, NC = L.nc;
    const int c0 = (int)r * NC;                           // first column of X held here
    const int ncols = max(0, min(NC, n - c0));            // columns of X held here
    const int kx = (m + 15) / 16;                         // K steps of the apply (rows of X)
    const AbortCtl ab{&ctl->abort_flag, 0u};              // timeouts stay in this CTA (it keeps to the barriers)

    griddep_launch_dependents();
    if (threadIdx.x == 0) {
        mbar_init(&ctl->load, 1);
        mbar_init(&ctl->mma, 1);
        ctl->abort_flag = 0;
        ctl->commits = 0;
        ctl->waited = 0;
        fence_barrier_init();
        prefetch_tensormap(&L.mapX);
    }
    if (warp == 0) {
        tmem_alloc(&ctl->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    griddep_wait();  // X and the scales come from the kernels before

    // ---- load this CTA's block of X once (rows >= m and columns >= n read as zero)
    const int npanels = (ncols + 63) / 64;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&ctl->load, (uint32_t)npanels * kPanel);
        for (int p = 0; p < npanels; ++p) tma_load_3d(Xs + p * kPanel, &L.mapX, &ctl->load, c0 + 64 * p, 0, u);
    }
    bool ok = true;
    if (lane == 0 && !mbar_wait_ctl(&ctl->load, 0, ab, L.wait_limit_ns, L.status)) ok = false;
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;

    const float s = L.scale[u];
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;  // the row of every TMEM read of this thread
    uint32_t mma_phase = 0;
    // issue one batch of MMAs (one thread), commit it, and wait (all threads)
    auto run_mma = [&](bool gram) {
        __syncthreads();
        if (threadIdx.x == 0 && !ctl->abort_flag) {
            tc_fence_after();
            if (gram) {
                constexpr uint32_t IDESC = idesc_bf16_f32(kRows, kRows, 0);
                const int ksteps = (ncols + 15) / 16;
                for (int k = 0; k < ksteps; ++k) {
                    const uint32_t a = smem_u32(Xs) + (uint32_t)(k >> 2) * kPanel + (uint32_t)(k & 3) * 32u;
                    const uint64_t d = smem_desc_sw128(a, 16, 1024);
                    tc_mma_f16(tmem, d, d, IDESC, k ? 1u : 0u);
                }
            } else {
                // D[128 x NC] = B (K-major, 128 x 128) * X_r (MN-major: K = rows of X), in 256-column halves
                constexpr uint32_t IDESC = idesc_bf16_f32(kRows, 256, 1);
                for (int h = 0; h * 256 < ncols; ++h) {
                    for (int k = 0; k < kx; ++k) {
                        const uint32_t a = smem_u32(Bs) + (uint32_t)(k >> 2) * kPanel + (uint32_t)(k & 3) * 32u;
                        const uint32_t b = smem_u32(Xs) + (uint32_t)h * 4u * kPanel + (uint32_t)k * (16u * 128u);
                        tc_mma_f16(tmem + (uint32_t)h * 256u, smem_desc_sw128(a, 16, 1024),
                                   smem_desc_sw128(b, kPanel, 1024), IDESC, k ? 1u : 0u);
                    }
                }
            }
            tc_commit(&ctl->mma);
            ctl->commits = ctl->commits + 1;
        }
        __syncthreads();
        bool good = !ctl->abort_flag;
        if (good && lane == 0) good = mbar_wait_ctl(&ctl->mma, mma_phase, ab, L.wait_limit_ns, L.status);
        if (good && threadIdx.x == 0) ctl->waited = ctl->waited + 1;
        good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
        mma_phase ^= 1u;
        tc_fence_after();
        return good;
    };

    for (int it = 0; it < L.steps; ++it) {
        const float a_k = L.coef[it][0], b_k = L.coef[it][1];
        const bool first = it == 0, last = it + 1 == L.steps;
        // ---- Gram partial A_r = X_r X_r^T, then its rows go to their reducers
        ok = run_mma(true) && ok;
        if (ok) {
            // thread: TMEM lane `row`, columns [64*half, 64*half + 64)
            const int d = row / kSlabRows;  // the CTA that reduces this row
            const uint32_t dst = mapa_shared(smem_u32(Rx), (uint32_t)d) + r * kSlab +
                                 (uint32_t)(row % kSlabRows) * (kRows * 4u);
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                float v[32];
                tmem_ld32(tmem + (uint32_t)(64 * half + 32 * c) + ((uint32_t)(quad * 32) << 16), v);
                if (ncols == 0) {  // no MMA wrote the accumulator: this CTA's partial is zero
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] = 0.f;
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint4 w;
                    w.x = __float_as_uint(v[4 * q]);
                    w.y = __float_as_uint(v[4 * q + 1]);
                    w.z = __float_as_uint(v[4 * q + 2]);
                    w.w = __float_as_uint(v[4 * q + 3]);
                    st_cluster_v4(dst + (uint32_t)(64 * half + 32 * c + 4 * q) * 4u, w);
                }
            }
        }
        tc_fence_before();
        cluster_sync_all();  // every partial is in its reducer's buffer
        // ---- reduce this CTA's 16 rows over the sources in order, scale, round,
        // and write them into every CTA's B
        {
            const int rr = threadIdx.x >> 4;          // row within the slab
            const int cc = (threadIdx.x & 15) * 8;    // 8 columns
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 1
            for (int src = 0; src < kCl; ++src) {
                const float4* p =
                    reinterpret_cast<const float4*>(Rx + src * kSlab + rr * (kRows * 4) + cc * 4);
                const float4 x0 = p[0], x1 = p[1];
                acc[0] += x0.x; acc[1] += x0.y; acc[2] += x0.z; acc[3] += x0.w;
                acc[4] += x1.x; acc[5] += x1.y; acc[6] += x1.z; acc[7] += x1.w;
            }
            const float coef = first ? b_k * s * s : b_k;
            uint4 w;
            w.x = pack_bf16x2(coef * acc[0], coef * acc[1]);
            w.y = pack_bf16x2(coef * acc[2], coef * acc[3]);
            w.z = pack_bf16x2(coef * acc[4], coef * acc[5]);
            w.w = pack_bf16x2(coef * acc[6], coef * acc[7]);
            const int grow = (int)r * kSlabRows + rr;  // row of A (and B)
            const uint32_t off = panel_off(grow, cc);
#pragma unroll 1
            for (int dst = 0; dst < kCl; ++dst) st_cluster_v4(mapa_shared(smem_u32(Bs) + off, (uint32_t)dst), w);
            fence_proxy_async_cluster();
        }
        cluster_sync_all();  // B is complete in every CTA
        fence_proxy_async_smem();
        // ---- apply: D = B X_r; X_r' = s*(a X_r + D), or the update of W
        ok = run_mma(false) && ok;
        if (ok) {
            const float sa = first ? s : 1.f;
            const float ca = sa * a_k;
            // this thread: row `row`, columns [NC/2 * half, NC/2 * (half + 1)) of the block, 32 at a time
            const int hc = NC / 2;
#pragma unroll 1
            for (int cb = half * hc; cb < (half + 1) * hc && cb < ncols; cb += 32) {
                float v[32];
                tmem_ld32(tmem + (uint32_t)cb + ((uint32_t)(quad * 32) << 16), v);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t o = (uint32_t)(cb >> 6) * kPanel + (uint32_t)row * 128u +
                                       ((((uint32_t)((cb & 63) >> 3) + q) ^ (uint32_t)(row & 7)) << 4);
                    const uint4 x = *reinterpret_cast<const uint4*>(Xs + o);
                    const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        v[8 * q + 2 * e] = ca * bf16_lo(xv[e]) + sa * v[8 * q + 2 * e];
                        v[8 * q + 2 * e + 1] = ca * bf16_hi(xv[e]) + sa * v[8 * q + 2 * e + 1];
                    }
                }
                if (!last) {
                    if (row < m) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint32_t o = (uint32_t)(cb >> 6) * kPanel + (uint32_t)row * 128u +
                                               ((((uint32_t)((cb & 63) >> 3) + q) ^ (uint32_t)(row & 7)) << 4);
                            uint4 w;
                            w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
                            w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
                            w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
                            w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
                            *reinterpret_cast<uint4*>(Xs + o) = w;
                        }
                    }
                } else if (row < m) {
                    // W row (head slice h of matrix bidx): 32 consecutive weights, 16 bytes at a time
                    const int bidx = u / L.heads, h = u - bidx * L.heads;
                    float* wrow = L.W[bidx] + ((int64_t)h * L.Rh + row) * L.C + c0 + cb;
                    const int left = min(32, ncols - cb);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (4 * q < left) {
                            float4 w = *reinterpret_cast<const float4*>(wrow + 4 * q);
                            w.x = update_w(w.x, v[4 * q + 0], L.decay, L.lr_s, L.lr_wd, L.cautious);
                            w.y = update_w(w.y, v[4 * q + 1], L.decay, L.lr_s, L.lr_wd, L.cautious);
                            w.z = update_w(w.z, v[4 * q + 2], L.decay, L.lr_s, L.lr_wd, L.cautious);
                            w.w = update_w(w.w, v[4 * q + 3], L.decay, L.lr_s, L.lr_wd, L.cautious);
                            *reinterpret_cast<float4*>(wrow + 4 * q) = w;
                        }
                    }
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();  // the new X is read by the next Gram's MMAs
    }

    // ---- wind down: after a timeout, wait (bounded, whatever the abort) for
    // the last MMA batch and for the load of X before TMEM is released
    __syncthreads();
    if (threadIdx.x == 0 && ctl->abort_flag) {
        const long long lim = L.wait_limit_ns > kDrainNs ? L.wait_limit_ns : kDrainNs;
        mbar_wait_ctl(&ctl->load, 0, ab, lim, L.status, 0, false, true);
        // every committed batch whose completion was not seen yet, in order
        // (at most the last one: no MMA is issued after an abort)
        for (int ph = ctl->waited; ph < ctl->commits; ++ph)
            mbar_wait_ctl(&ctl->mma, (uint32_t)(ph & 1), ab, lim, L.status, 0, false, true);
    }
    __syncwarp();
    __syncthreads();
    tc_fence_before();
    cluster_sync_all();  // no CTA leaves while another may still write into its shared memory
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_cluster() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(ptr);
        return nullptr;
    }();
    return fn;
}

}  // namespace

bool ns_cluster_eligible(int m, int n, int transposed) {
    return m >= 1 && m <= kRows && !transposed && n >= 1 && n <= kCl * kMaxNC;
}

int ns_cluster_cols(int n) {
    const int per = (n + kCl - 1) / kCl;
    return (per + 63) / 64 * 64;
}

cudaError_t ns_cluster_setup() {
    static PerDevice<int> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int done = 0;
    return cache.get(dev, &done, [](int* v) -> cudaError_t {
        const cudaError_t r =
            cudaFuncSetAttribute(ns_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
        *v = 1;
        return r;
    });
}

cudaError_t launch_ns_cluster(const NsClusterIn& in, cudaStream_t s) {
    if (!ns_cluster_eligible(in.m, in.n, 0) || in.units < 1 || in.steps < 1 || in.steps > MA_MAX_NS_STEPS ||
        in.heads < 1 || in.units / in.heads > MA_MAX_BATCH)
        return cudaErrorInvalidValue;
    EncodeTiledFn enc = encode_fn_cluster();
    if (!enc) return cudaErrorNotSupported;
    cudaError_t e = ns_cluster_setup();
    if (e != cudaSuccess) return e;
    static thread_local NsClusterLaunch L;
    std::memset(&L, 0, sizeof(L));
    // X: [units][m][ldx] bf16, boxes of 64 columns x 128 rows (rows >= m and columns >= n read as zero)
    cuuint64_t dims[3] = {(cuuint64_t)in.n, (cuuint64_t)in.m, (cuuint64_t)in.units};
    cuuint64_t strides[2] = {(cuuint64_t)in.ldx * 2, (cuuint64_t)in.x_unit * 2};
    cuuint32_t box[3] = {64, kRows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&L.mapX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(in.x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    L.m = in.m;
    L.n = in.n;
    L.nc = ns_cluster_cols(in.n);
    L.steps = in.steps;
    for (int k = 0; k < in.steps; ++k) {
        L.coef[k][0] = in.coef[k][0];
        L.coef[k][1] = in.coef[k][1];
    }
    L.scale = in.scale;
    L.heads = in.heads;
    L.Rh = in.Rh;
    L.C = in.C;
    L.decay = in.decay;
    L.lr_s = in.lr_s;
    L.lr_wd = in.lr_wd;
    L.cautious = in.cautious;
    L.wait_limit_ns = in.wait_limit_ns;
    L.status = in.status;
    for (int b = 0; b < in.units / in.heads; ++b) L.W[b] = in.W[b];
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = MA_PDL;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(kCl * in.units));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ns_cluster_kernel, L);
}

bool ns_cluster_is_kernel(const void* func) { return func == reinterpret_cast<const void*>(ns_cluster_kernel); }

size_t ns_cluster_launch_bytes() { return sizeof(NsClusterLaunch); }

int ns_cluster_patch(void* launch, NsFinalPatchFn f, void* ctx) {
    NsClusterLaunch* L = reinterpret_cast<NsClusterLaunch*>(launch);
    return f(ctx, L->W[0], L->Rh, L->C, &L->decay, &L->lr_s, &L->lr_wd);
}

}  // namespace ma
