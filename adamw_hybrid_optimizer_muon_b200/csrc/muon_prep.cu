// Muon momentum, Nesterov direction and Frobenius norm, in one HBM pass.
//
// "MuonClip Optimizer", "Momentum": m <- beta*m + (1-beta)*g (EMA, decay
// 0.95). With Nesterov ("How nanochat Combines Muon and AdamW in a Single
// Optimizer", "Muon Step Implementation") the direction is
// u = beta*m + (1-beta)*g, otherwise u = m. As in the muown_triton `_prepare`
// contract, momentum is mutated in place, the gradient is preserved, and the
// operand for the orthogonalisation is emitted as bf16 (fp32 in precision
// mode 1).
//
// The kernel also writes one partial sum of u^2 per block, taken from the fp32
// u before rounding. The finalize kernel adds the partials of each unit (a
// matrix, or one head slice of it) in a fixed order and stores
// 1/(||u||_F + eps), the Frobenius normalisation that the Newton-Schulz GEMMs
// fold into their epilogues. The sum is deterministic: no float atomics.
//
// Bytes per element: g 2 (bf16) + m read 4 + m write 4 + X write 2 = 12.
//
// Two layouts:
//  * flat: the unit is wide (rows <= cols), so X is u itself (row stride C).
//    Each thread streams 8 elements per iteration with 16-byte accesses.
//  * transposing: the unit is tall (rows > cols), so X = u^T. 64x64 tiles go
//    through shared memory, and reads and writes are both coalesced.
#include "common.cuh"
#include "internal.h"

namespace ma {

namespace {

// Sum of v over the block's NT threads in a fixed order (a butterfly within
// each warp, then the warps in order); thread 0 gets it. `red` may be reused
// by the next call, hence the trailing barrier.
template <int NT>
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    float t = 0.f;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < NT / 32; ++i) t += red[i];
    }
    __syncthreads();
    return t;
}

template <bool GBF16>
__device__ __forceinline__ void load_g8(const void* G, int64_t i, float (&g)[8]) {
    if (GBF16) {
        const uint4 w = __ldcs(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(G) + i));
        g[0] = bf16_lo(w.x); g[1] = bf16_hi(w.x); g[2] = bf16_lo(w.y); g[3] = bf16_hi(w.y);
        g[4] = bf16_lo(w.z); g[5] = bf16_hi(w.z); g[6] = bf16_lo(w.w); g[7] = bf16_hi(w.w);
    } else {
        const float4* gp = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(G) + i);
        const float4 a = __ldcs(gp), c = __ldcs(gp + 1);
        g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w; g[4] = c.x; g[5] = c.y; g[6] = c.z; g[7] = c.w;
    }
}

// m <- beta*m + (1-beta)*g on 8 elements; d <- the direction; returns sum of d^2.
__device__ __forceinline__ float momentum8(float (&m)[8], const float (&g)[8], float (&d)[8], float beta, float omb,
                                           bool nesterov) {
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        m[k] = beta * m[k] + omb * g[k];
        d[k] = nesterov ? beta * m[k] + omb * g[k] : m[k];
        ss += d[k] * d[k];
    }
    return ss;
}

template <bool XF32>
__device__ __forceinline__ void store_x8(void* X, int64_t i, const float (&d)[8]) {
    if (XF32) {
        float4* xp = reinterpret_cast<float4*>(reinterpret_cast<float*>(X) + i);
        __stcs(xp, make_float4(d[0], d[1], d[2], d[3]));
        __stcs(xp + 1, make_float4(d[4], d[5], d[6], d[7]));
    } else {
        uint4 w;
        w.x = pack_bf16x2(d[0], d[1]);
        w.y = pack_bf16x2(d[2], d[3]);
        w.z = pack_bf16x2(d[4], d[5]);
        w.w = pack_bf16x2(d[6], d[7]);
        __stcs(reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(X) + i), w);
    }
}

// The chunk of a flat unit that one 256-thread block of prep_flat_kernel
// covers: pass vt (0..255) handles the 8-element groups vt, vt + 256, ...;
// returns its sum of squares, accumulated in that order. Loads for a full
// chunk are all issued before any arithmetic (12 independent 16-byte loads
// in flight per pass).
template <bool GBF16, bool XF32>
__device__ __forceinline__ float prep_flat_pass(const MuonPrepLaunch& L, int u, int64_t part, int vt) {
    constexpr int kIter = kPrepChunk / (8 * 256);
    const int b = u / L.heads, h = u % L.heads;
    const int64_t unit_elems = L.Rh * L.C;
    const int64_t off = (int64_t)h * unit_elems;
    const int64_t start = part * kPrepChunk;
    const int64_t end = min(start + (int64_t)kPrepChunk, unit_elems);
    float* M = L.M[b] + off;
    const void* G = GBF16 ? static_cast<const void*>(reinterpret_cast<const uint16_t*>(L.G[b]) + off)
                          : static_cast<const void*>(reinterpret_cast<const float*>(L.G[b]) + off);
    void* X = XF32 ? static_cast<void*>(reinterpret_cast<float*>(L.X) + (int64_t)u * L.x_unit)
                   : static_cast<void*>(reinterpret_cast<uint16_t*>(L.X) + (int64_t)u * L.x_unit);
    const float beta = L.beta, omb = L.omb;
    const bool nest = L.nesterov != 0;
    // buffer extents for the guarded build: a matrix's G and M, and the workspace's X
    [[maybe_unused]] const int64_t mat_elems = (int64_t)L.heads * unit_elems;
    [[maybe_unused]] const int64_t x_elems = (int64_t)L.batch * L.heads * L.x_unit;
    [[maybe_unused]] const int64_t xu = (int64_t)u * L.x_unit;
    float ss = 0.f;
    if (end - start == kPrepChunk) {
        float g[kIter][8], m[kIter][8];
        bool ok[kIter];
#pragma unroll
        for (int k = 0; k < kIter; ++k) {
            const int64_t i = start + 8 * ((int64_t)k * 256 + vt);
            ok[k] = MA_INB(off + i, 8, mat_elems, L.status) && MA_INB(xu + i, 8, x_elems, L.status);
#pragma unroll
            for (int e = 0; e < 8; ++e) g[k][e] = m[k][e] = 0.f;
            if (!ok[k]) continue;
            load_g8<GBF16>(G, i, g[k]);
            const float4 a = __ldcs(reinterpret_cast<const float4*>(M + i));
            const float4 c = __ldcs(reinterpret_cast<const float4*>(M + i + 4));
            m[k][0] = a.x; m[k][1] = a.y; m[k][2] = a.z; m[k][3] = a.w;
            m[k][4] = c.x; m[k][5] = c.y; m[k][6] = c.z; m[k][7] = c.w;
        }
#pragma unroll
        for (int k = 0; k < kIter; ++k) {
            const int64_t i = start + 8 * ((int64_t)k * 256 + vt);
            float d[8];
            ss += momentum8(m[k], g[k], d, beta, omb, nest);
            if (!ok[k]) continue;
            __stcs(reinterpret_cast<float4*>(M + i), make_float4(m[k][0], m[k][1], m[k][2], m[k][3]));
            __stcs(reinterpret_cast<float4*>(M + i + 4), make_float4(m[k][4], m[k][5], m[k][6], m[k][7]));
            store_x8<XF32>(X, i, d);
        }
    } else {
        for (int64_t i = start + 8 * (int64_t)vt; i < end; i += 8 * 256) {
            if (!(MA_INB(off + i, 8, mat_elems, L.status) && MA_INB(xu + i, 8, x_elems, L.status))) continue;
            float g[8], m[8], d[8];
            load_g8<GBF16>(G, i, g);
            const float4 a = __ldcs(reinterpret_cast<const float4*>(M + i));
            const float4 c = __ldcs(reinterpret_cast<const float4*>(M + i + 4));
            m[0] = a.x; m[1] = a.y; m[2] = a.z; m[3] = a.w; m[4] = c.x; m[5] = c.y; m[6] = c.z; m[7] = c.w;
            ss += momentum8(m, g, d, beta, omb, nest);
            __stcs(reinterpret_cast<float4*>(M + i), make_float4(m[0], m[1], m[2], m[3]));
            __stcs(reinterpret_cast<float4*>(M + i + 4), make_float4(m[4], m[5], m[6], m[7]));
            store_x8<XF32>(X, i, d);
        }
    }
    return ss;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Flat path, on the caller's stream: one block of 256 threads per chunk of
// kPrepChunk elements of one unit. The chunk's partial is the sum over the
// block in a fixed order: each warp's butterfly, then the eight warps in order.
template <bool GBF16, bool XF32>
__global__ void __launch_bounds__(256) prep_flat_kernel(const __grid_constant__ MuonPrepLaunch L) {
    griddep_launch_dependents();
    griddep_wait();
    __shared__ float red[8];
    const int u = blockIdx.y;
    const float s = warp_sum(prep_flat_pass<GBF16, XF32>(L, u, blockIdx.x, threadIdx.x));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += red[w];
        L.partials[(int64_t)u * L.parts + blockIdx.x] = (double)t;
    }
}

// Flat path under another batch's Newton-Schulz kernels (a side stream): a
// small grid of kPrepSideThreads-thread blocks walks the (unit, chunk) pairs
// grid-stride. At most 85 registers a thread and 32 bytes of shared memory:
// a block fits on an SM beside a Newton-Schulz CTA. Each thread makes the
// passes of two of prep_flat_kernel's threads (vt and vt + 128, one after the
// other) and keeps their sums apart, and the warps' butterflies and the final
// sum run in prep_flat_kernel's order: every partial, and so every scale, is
// the same bits on either path.
template <bool GBF16, bool XF32>
__global__ void __launch_bounds__(kPrepSideThreads, 6) prep_flat_side_kernel(const __grid_constant__ MuonPrepLaunch L) {
    griddep_launch_dependents();
    griddep_wait();
    __shared__ float red[8];
    const int64_t items = (int64_t)L.batch * L.heads * L.parts;
    const int w = threadIdx.x >> 5;
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
        const int u = (int)(it / L.parts);
        const int64_t part = it - (int64_t)u * L.parts;
        const float lo = warp_sum(prep_flat_pass<GBF16, XF32>(L, u, part, threadIdx.x));        // warps 0..3
        const float hi = warp_sum(prep_flat_pass<GBF16, XF32>(L, u, part, threadIdx.x + 128));  // warps 4..7
        if ((threadIdx.x & 31) == 0) {
            red[w] = lo;
            red[4 + w] = hi;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            float t = 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q) t += red[q];
            L.partials[(int64_t)u * L.parts + part] = (double)t;
        }
        __syncthreads();  // red is reused by the next chunk
    }
}

// Transposing path (tall units, X = u^T), without shared memory: a block
// takes a 64-row x 64-column block of u, warp w its rows 16w .. 16w + 15 and
// lane l columns 2l and 2l + 1. Row by row a warp reads 256 bytes of momentum
// and 128 of bf16 gradient as 8- and 4-byte vectors, all sixteen rows' loads
// in flight before any arithmetic (fp32 gradients: two batches of eight);
// the direction overwrites the momentum in registers once the new momentum
// has gone out. Lane l then holds 16 consecutive elements of rows c0 + 2l
// and c0 + 2l + 1 of X: one whole 32-byte sector each (bf16), which the four
// warps of the block complete to whole 128-byte lines. The block's partial
// is the warps' sums in order, each a butterfly over lanes that added their
// 32 values row by row. Blocks walk the (unit, block) pairs grid-stride: one
// block per pair on the caller's stream, or a small grid on a side stream,
// where a block (at most 80 registers a thread, 16 bytes of shared memory)
// fits beside a Newton-Schulz CTA. The partials do not depend on the grid.
template <bool GBF16, bool XF32>
__global__ void __launch_bounds__(kPrepSideThreads, 6) prep_transpose_kernel(const __grid_constant__ MuonPrepLaunch L) {
    griddep_launch_dependents();
    griddep_wait();
    constexpr int RW = kPrepTRows / (kPrepSideThreads / 32);  // rows per warp
    static_assert(RW == 16 && kPrepTCols == 2 * 32, "block shape");
    constexpr int RB = GBF16 ? RW : RW / 2;  // rows whose loads are in flight together
    constexpr int GW = GBF16 ? 1 : 2;        // gradient words per row and lane
    __shared__ float red[kPrepSideThreads / 32];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t items = (int64_t)L.batch * L.heads * L.parts;
    const float beta = L.beta, omb = L.omb;
    const bool nest = L.nesterov != 0;
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
        const int u = (int)(it / L.parts);
        const int64_t part = it - (int64_t)u * L.parts;
        const int b = u / L.heads, h = u % L.heads;
        const int64_t off = (int64_t)h * L.Rh * L.C;
        const int64_t r0 = (part / L.tiles_c) * kPrepTRows + RW * w;  // this warp's first row of u
        const int64_t c = (part % L.tiles_c) * kPrepTCols + 2 * lane;  // this lane's first column of u
        // C % 8 == 0: a lane's two columns are both in range or both out of it
        const int rows = c < L.C ? (int)max((int64_t)0, min((int64_t)RW, L.Rh - r0)) : 0;
        const int64_t e0 = off + r0 * L.C + c;  // element index of (r0, c)
        // buffer extents for the guarded build: a matrix's G and M, and the workspace's X
        [[maybe_unused]] const int64_t mat_elems = (int64_t)L.heads * L.Rh * L.C;
        [[maybe_unused]] const int64_t x_elems = (int64_t)L.batch * L.heads * L.x_unit;
        float* mp = L.M[b] + e0;
        const uint32_t* gp = reinterpret_cast<const uint32_t*>(L.G[b]) + (GBF16 ? e0 / 2 : e0);
        const int64_t gstride = GBF16 ? L.C / 2 : L.C;  // words per row
        float d[RW][2];  // momentum in, then the direction
        float ss = 0.f;
#pragma unroll
        for (int i0 = 0; i0 < RW; i0 += RB) {
            uint32_t g[RB][GW];
#pragma unroll
            for (int i = i0; i < i0 + RB; ++i) {
                d[i][0] = d[i][1] = 0.f;
#pragma unroll
                for (int k = 0; k < GW; ++k) g[i - i0][k] = 0u;
                if (i < rows && MA_INB(e0 + (int64_t)i * L.C, 2, mat_elems, L.status)) {
                    const float2 mv = __ldcs(reinterpret_cast<const float2*>(mp + (int64_t)i * L.C));
                    d[i][0] = mv.x;
                    d[i][1] = mv.y;
                    if (GBF16) {
                        g[i - i0][0] = __ldcs(gp + (int64_t)i * gstride);
                    } else {
                        const uint2 gv = __ldcs(reinterpret_cast<const uint2*>(gp + (int64_t)i * gstride));
                        g[i - i0][0] = gv.x;
                        g[i - i0][GW - 1] = gv.y;
                    }
                }
            }
#pragma unroll
            for (int i = i0; i < i0 + RB; ++i) {
                if (i < rows && MA_INB(e0 + (int64_t)i * L.C, 2, mat_elems, L.status)) {
                    const float g0 = GBF16 ? bf16_lo(g[i - i0][0]) : __uint_as_float(g[i - i0][0]);
                    const float g1 = GBF16 ? bf16_hi(g[i - i0][0]) : __uint_as_float(g[i - i0][GW - 1]);
                    const float mn0 = beta * d[i][0] + omb * g0;
                    const float mn1 = beta * d[i][1] + omb * g1;
                    d[i][0] = nest ? beta * mn0 + omb * g0 : mn0;
                    d[i][1] = nest ? beta * mn1 + omb * g1 : mn1;
                    ss += d[i][0] * d[i][0];
                    ss += d[i][1] * d[i][1];
                    __stcs(reinterpret_cast<float2*>(mp + (int64_t)i * L.C), make_float2(mn0, mn1));
                }
            }
        }
        // rows c and c + 1 of X, elements r0 .. r0 + 15
        if (rows > 0) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int64_t xi = (int64_t)u * L.x_unit + (c + j) * L.ldx + r0;
                if (!MA_INB(xi, rows, x_elems, L.status)) continue;
                if (rows == RW) {
                    if (XF32) {
                        float4* xp = reinterpret_cast<float4*>(reinterpret_cast<float*>(L.X) + xi);
#pragma unroll
                        for (int q = 0; q < RW / 4; ++q)
                            __stcs(xp + q, make_float4(d[4 * q][j], d[4 * q + 1][j], d[4 * q + 2][j], d[4 * q + 3][j]));
                    } else {
                        uint4* xp = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(L.X) + xi);
#pragma unroll
                        for (int q = 0; q < RW / 8; ++q) {
                            uint4 v;
                            v.x = pack_bf16x2(d[8 * q + 0][j], d[8 * q + 1][j]);
                            v.y = pack_bf16x2(d[8 * q + 2][j], d[8 * q + 3][j]);
                            v.z = pack_bf16x2(d[8 * q + 4][j], d[8 * q + 5][j]);
                            v.w = pack_bf16x2(d[8 * q + 6][j], d[8 * q + 7][j]);
                            __stcs(xp + q, v);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < RW; ++i) {
                        if (i < rows) {
                            if (XF32) reinterpret_cast<float*>(L.X)[xi + i] = d[i][j];
                            else reinterpret_cast<__nv_bfloat16*>(L.X)[xi + i] = __float2bfloat16_rn(d[i][j]);
                        }
                    }
                }
            }
        }
        const float tot = block_sum<kPrepSideThreads>(ss, red);
        if (threadIdx.x == 0) L.partials[(int64_t)u * L.parts + part] = (double)tot;
    }
}

// One warp per unit: lane-strided sum of the unit's partials, then a fixed
// butterfly, so the result does not depend on scheduling.
__global__ void __launch_bounds__(256) norm_finalize_kernel(const double* __restrict__ partials, int64_t parts,
                                                            int units, float eps, float* __restrict__ scale) {
    griddep_launch_dependents();
    griddep_wait();
    const int u = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int l = threadIdx.x & 31;
    if (u >= units) return;
    double s = 0.0;
    for (int64_t i = l; i < parts; i += 32) s += partials[(int64_t)u * parts + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (l == 0) scale[u] = (float)(1.0 / (sqrt(s) + (double)eps));
}

}  // namespace

int64_t prep_parts_per_unit(int64_t Rh, int64_t C, int transposed) {
    if (transposed) return ((Rh + kPrepTRows - 1) / kPrepTRows) * ((C + kPrepTCols - 1) / kPrepTCols);
    return (Rh * C + kPrepChunk - 1) / kPrepChunk;
}

// The kernels that run beside Newton-Schulz CTAs prefer the largest
// shared-memory carveout, the one those CTAs set on their SMs, so that their
// blocks can join those SMs.
// Once per device; the attribute is set before any stream capture by the
// library's set-up (the first call on a device).
cudaError_t prep_setup() {
    static PerDevice<int> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int done = 0;
    return cache.get(dev, &done, [](int* v) -> cudaError_t {
        const void* fns[8] = {reinterpret_cast<const void*>(prep_flat_side_kernel<true, false>),
                              reinterpret_cast<const void*>(prep_flat_side_kernel<true, true>),
                              reinterpret_cast<const void*>(prep_flat_side_kernel<false, false>),
                              reinterpret_cast<const void*>(prep_flat_side_kernel<false, true>),
                              reinterpret_cast<const void*>(prep_transpose_kernel<true, false>),
                              reinterpret_cast<const void*>(prep_transpose_kernel<true, true>),
                              reinterpret_cast<const void*>(prep_transpose_kernel<false, false>),
                              reinterpret_cast<const void*>(prep_transpose_kernel<false, true>)};
        for (const void* f : fns) {
            const cudaError_t r = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                                       cudaSharedmemCarveoutMaxShared);
            if (r != cudaSuccess) return r;
        }
        *v = 1;
        return cudaSuccess;
    });
}

cudaError_t launch_muon_prep(const MuonPrepLaunch& L, int max_blocks, cudaStream_t s) {
    const int units = L.batch * L.heads;
    if (units == 0 || L.parts == 0) return cudaSuccess;
    const bool gb = L.gdt == MA_BF16, xf = L.x_f32 != 0;
    cudaError_t e;
    if (L.transposed) {
        if ((e = prep_setup()) != cudaSuccess) return e;
        int64_t items = (int64_t)units * L.parts;
        if (max_blocks > 0 && items > max_blocks) items = max_blocks;
        if (items > INT32_MAX) items = INT32_MAX;
        const dim3 grid((unsigned)items), block(kPrepSideThreads);
        if (gb && !xf) e = launch_pdl(prep_transpose_kernel<true, false>, grid, block, 0, s, L);
        else if (gb) e = launch_pdl(prep_transpose_kernel<true, true>, grid, block, 0, s, L);
        else if (!xf) e = launch_pdl(prep_transpose_kernel<false, false>, grid, block, 0, s, L);
        else e = launch_pdl(prep_transpose_kernel<false, true>, grid, block, 0, s, L);
    } else if (max_blocks <= 0) {
        const dim3 grid((unsigned)L.parts, (unsigned)units);
        if (gb && !xf) e = launch_pdl(prep_flat_kernel<true, false>, grid, dim3(256), 0, s, L);
        else if (gb) e = launch_pdl(prep_flat_kernel<true, true>, grid, dim3(256), 0, s, L);
        else if (!xf) e = launch_pdl(prep_flat_kernel<false, false>, grid, dim3(256), 0, s, L);
        else e = launch_pdl(prep_flat_kernel<false, true>, grid, dim3(256), 0, s, L);
    } else {
        if ((e = prep_setup()) != cudaSuccess) return e;
        int64_t items = (int64_t)units * L.parts;
        if (items > max_blocks) items = max_blocks;
        const dim3 grid((unsigned)items), block(kPrepSideThreads);
        if (gb && !xf) e = launch_pdl(prep_flat_side_kernel<true, false>, grid, block, 0, s, L);
        else if (gb) e = launch_pdl(prep_flat_side_kernel<true, true>, grid, block, 0, s, L);
        else if (!xf) e = launch_pdl(prep_flat_side_kernel<false, false>, grid, block, 0, s, L);
        else e = launch_pdl(prep_flat_side_kernel<false, true>, grid, block, 0, s, L);
    }
    return e;
}

cudaError_t launch_norm_finalize(const double* partials, int64_t parts, int units, float eps, float* scale,
                                 cudaStream_t s) {
    if (units == 0) return cudaSuccess;
    return launch_pdl(norm_finalize_kernel, dim3((units + 7) / 8), dim3(256), 0, s, partials, parts, units, eps,
                      scale);
}

}  // namespace ma
