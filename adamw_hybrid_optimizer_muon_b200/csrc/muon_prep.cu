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

__device__ __forceinline__ float block_sum_256(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    float t = 0.f;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) t += red[i];
    }
    return t;
}

__global__ void __launch_bounds__(256) prep_flat_kernel(const __grid_constant__ MuonPrepLaunch L) {
    __shared__ float red[8];
    const int u = blockIdx.y;
    const int b = u / L.heads, h = u % L.heads;
    const int64_t unit_elems = L.Rh * L.C;
    const int64_t off = (int64_t)h * unit_elems;
    const int64_t start = (int64_t)blockIdx.x * kPrepChunk;
    const int64_t end = min(start + (int64_t)kPrepChunk, unit_elems);
    float* M = L.M[b] + off;
    const float beta = L.beta, omb = L.omb;
    float ss = 0.f;
    for (int64_t i = start + 8 * (int64_t)threadIdx.x; i < end; i += 8 * 256) {
        float g[8];
        if (L.gdt == MA_BF16) {
            const uint4 w = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(L.G[b]) + off + i);
            g[0] = bf16_lo(w.x); g[1] = bf16_hi(w.x); g[2] = bf16_lo(w.y); g[3] = bf16_hi(w.y);
            g[4] = bf16_lo(w.z); g[5] = bf16_hi(w.z); g[6] = bf16_lo(w.w); g[7] = bf16_hi(w.w);
        } else {
            const float* gp = reinterpret_cast<const float*>(L.G[b]) + off + i;
            const float4 a = *reinterpret_cast<const float4*>(gp);
            const float4 c = *reinterpret_cast<const float4*>(gp + 4);
            g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w; g[4] = c.x; g[5] = c.y; g[6] = c.z; g[7] = c.w;
        }
        float4 m0 = *reinterpret_cast<const float4*>(M + i);
        float4 m1 = *reinterpret_cast<const float4*>(M + i + 4);
        float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
        float d[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            m[k] = beta * m[k] + omb * g[k];
            d[k] = L.nesterov ? beta * m[k] + omb * g[k] : m[k];
            ss += d[k] * d[k];
        }
        *reinterpret_cast<float4*>(M + i) = make_float4(m[0], m[1], m[2], m[3]);
        *reinterpret_cast<float4*>(M + i + 4) = make_float4(m[4], m[5], m[6], m[7]);
        if (L.x_f32) {
            float* X = reinterpret_cast<float*>(L.X) + (int64_t)u * L.x_unit + i;
            *reinterpret_cast<float4*>(X) = make_float4(d[0], d[1], d[2], d[3]);
            *reinterpret_cast<float4*>(X + 4) = make_float4(d[4], d[5], d[6], d[7]);
        } else {
            uint16_t* X = reinterpret_cast<uint16_t*>(L.X) + (int64_t)u * L.x_unit + i;
            uint4 w;
            w.x = pack_bf16x2(d[0], d[1]);
            w.y = pack_bf16x2(d[2], d[3]);
            w.z = pack_bf16x2(d[4], d[5]);
            w.w = pack_bf16x2(d[6], d[7]);
            *reinterpret_cast<uint4*>(X) = w;
        }
    }
    const float tot = block_sum_256(ss, red);
    if (threadIdx.x == 0) L.partials[(int64_t)u * L.parts + blockIdx.x] = (double)tot;
}

__global__ void __launch_bounds__(256) prep_transpose_kernel(const __grid_constant__ MuonPrepLaunch L) {
    __shared__ float tile[kPrepTile][kPrepTile + 1];
    __shared__ float red[8];
    const int u = blockIdx.y;
    const int b = u / L.heads, h = u % L.heads;
    const int64_t off = (int64_t)h * L.Rh * L.C;
    const int64_t tr = blockIdx.x / L.tiles_c, tc = blockIdx.x % L.tiles_c;
    const int64_t r0 = tr * kPrepTile, c0 = tc * kPrepTile;
    const int col = threadIdx.x & 63, rsub = threadIdx.x >> 6;
    float* M = L.M[b] + off;
    const float beta = L.beta, omb = L.omb;
    float ss = 0.f;
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
        const int rl = rsub + 4 * k;
        const int64_t r = r0 + rl, c = c0 + col;
        float d = 0.f;
        if (r < L.Rh && c < L.C) {
            const int64_t idx = r * L.C + c;
            float g;
            if (L.gdt == MA_BF16)
                g = __uint_as_float(uint32_t(reinterpret_cast<const uint16_t*>(L.G[b])[off + idx]) << 16);
            else
                g = reinterpret_cast<const float*>(L.G[b])[off + idx];
            float m = beta * M[idx] + omb * g;
            M[idx] = m;
            d = L.nesterov ? beta * m + omb * g : m;
            ss += d * d;
        }
        tile[rl][col] = d;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
        const int cl = rsub + 4 * k;
        const int64_t xr = c0 + cl, xc = r0 + col;  // X = u^T: row = original column
        if (xr < L.C && xc < L.Rh) {
            const float d = tile[col][cl];
            const int64_t xi = (int64_t)u * L.x_unit + xr * L.ldx + xc;
            if (L.x_f32) reinterpret_cast<float*>(L.X)[xi] = d;
            else reinterpret_cast<__nv_bfloat16*>(L.X)[xi] = __float2bfloat16_rn(d);
        }
    }
    const float tot = block_sum_256(ss, red);
    if (threadIdx.x == 0) L.partials[(int64_t)u * L.parts + blockIdx.x] = (double)tot;
}

// One warp per unit: lane-strided sum of the unit's partials, then a fixed
// butterfly, so the result does not depend on scheduling.
__global__ void __launch_bounds__(256) norm_finalize_kernel(const double* __restrict__ partials, int64_t parts,
                                                            int units, float eps, float* __restrict__ scale) {
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
    if (transposed) return ((Rh + kPrepTile - 1) / kPrepTile) * ((C + kPrepTile - 1) / kPrepTile);
    return (Rh * C + kPrepChunk - 1) / kPrepChunk;
}

cudaError_t launch_muon_prep(const MuonPrepLaunch& L, cudaStream_t s) {
    const int units = L.batch * L.heads;
    if (units == 0 || L.parts == 0) return cudaSuccess;
    dim3 grid((unsigned)L.parts, (unsigned)units);
    if (L.transposed) prep_transpose_kernel<<<grid, 256, 0, s>>>(L);
    else prep_flat_kernel<<<grid, 256, 0, s>>>(L);
    return cudaGetLastError();
}

cudaError_t launch_norm_finalize(const double* partials, int64_t parts, int units, float eps, float* scale,
                                 cudaStream_t s) {
    if (units == 0) return cudaSuccess;
    norm_finalize_kernel<<<(units + 7) / 8, 256, 0, s>>>(partials, parts, units, eps, scale);
    return cudaGetLastError();
}

}  // namespace ma
