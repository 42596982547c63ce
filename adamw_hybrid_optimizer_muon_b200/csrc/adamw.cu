// Multi-tensor AdamW (the AdamW half of MuonAdamW).
//
// Follows "How nanochat Combines Muon and AdamW in a Single Optimizer",
// "AdamW Step Implementation": first and second moments per element and
// decoupled weight decay. The bias corrections are runtime scalars, as in the
// muown_triton `_finish` contract (BC1, BC2, LR, WD). The host forms
// lr/(1-b1^t) and 1/sqrt(1-b2^t) in double, once per group.
//
// The pass is bound by HBM bandwidth. Per element it reads p, m, v (fp32) and
// g (bf16 or fp32) and writes p, m, v: 26 bytes with bf16 gradients, 28 with
// fp32. Each block owns one 8192-element chunk of one tensor. It finds the
// tensor by binary search over the chunk prefix in the parameter block, then
// streams the chunk with 16-byte loads and stores (4 elements per thread per
// iteration), so one launch covers every AdamW tensor of a step.
#include "common.cuh"
#include "internal.h"

namespace ma {

namespace {

__device__ __forceinline__ void adamw_elem(float& p, float& m, float& v, float g, const AdamwGroupConst& H) {
    m = H.beta1 * m + H.omb1 * g;
    v = H.beta2 * v + H.omb2 * (g * g);
    const float denom = sqrtf(v) * H.inv_sqrt_bc2 + H.eps;
    p = p * H.decay - H.step_size * (m / denom);
}

__device__ __forceinline__ void load_g4(const void* g, int gdt, int64_t i, float (&out)[4]) {
    if (gdt == MA_BF16) {
        const uint2 w = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(g) + i);
        out[0] = bf16_lo(w.x);
        out[1] = bf16_hi(w.x);
        out[2] = bf16_lo(w.y);
        out[3] = bf16_hi(w.y);
    } else {
        const float4 f = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(g) + i);
        out[0] = f.x;
        out[1] = f.y;
        out[2] = f.z;
        out[3] = f.w;
    }
}

__device__ __forceinline__ float load_g1(const void* g, int gdt, int64_t i) {
    if (gdt == MA_BF16) return __uint_as_float(uint32_t(reinterpret_cast<const uint16_t*>(g)[i]) << 16);
    return reinterpret_cast<const float*>(g)[i];
}

__global__ void __launch_bounds__(256) adamw_kernel(const __grid_constant__ AdamwLaunch L) {
    griddep_launch_dependents();
    griddep_wait();
    const int64_t chunk = blockIdx.x;
    int lo = 0, hi = L.ntensors - 1;
    while (lo < hi) {  // last tensor whose first chunk is <= this chunk
        const int mid = (lo + hi + 1) >> 1;
        if (L.t[mid].chunk0 <= chunk) lo = mid;
        else hi = mid - 1;
    }
    const AdamwTensorDesc& T = L.t[lo];
    const AdamwGroupConst H = L.grp[T.group];
    const int64_t start = (chunk - T.chunk0) * kAdamwChunk;
    if (start >= T.numel) return;
    const int64_t end = min(start + (int64_t)kAdamwChunk, T.numel);

    int64_t scalar_from = start;
    if (T.vec) {
        const int64_t nvec_end = start + ((end - start) & ~int64_t(3));
#pragma unroll 2
        for (int64_t i = start + 4 * (int64_t)threadIdx.x; i < nvec_end; i += 4 * 256) {
            if (!MA_INB(i, 4, T.numel, L.status)) continue;
            float4 p = *reinterpret_cast<const float4*>(T.p + i);
            float4 m = *reinterpret_cast<const float4*>(T.m + i);
            float4 v = *reinterpret_cast<const float4*>(T.v + i);
            float g[4];
            load_g4(T.g, L.gdt, i, g);
            adamw_elem(p.x, m.x, v.x, g[0], H);
            adamw_elem(p.y, m.y, v.y, g[1], H);
            adamw_elem(p.z, m.z, v.z, g[2], H);
            adamw_elem(p.w, m.w, v.w, g[3], H);
            *reinterpret_cast<float4*>(T.p + i) = p;
            *reinterpret_cast<float4*>(T.m + i) = m;
            *reinterpret_cast<float4*>(T.v + i) = v;
        }
        scalar_from = nvec_end;
    }
    for (int64_t i = scalar_from + threadIdx.x; i < end; i += 256) {
        if (!MA_INB(i, 1, T.numel, L.status)) continue;
        float p = T.p[i], m = T.m[i], v = T.v[i];
        adamw_elem(p, m, v, load_g1(T.g, L.gdt, i), H);
        T.p[i] = p;
        T.m[i] = m;
        T.v[i] = v;
    }
}

}  // namespace

const void* adamw_kernel_func() { return reinterpret_cast<const void*>(adamw_kernel); }

cudaError_t launch_adamw(const AdamwLaunch& L, cudaStream_t s) {
    if (L.nchunks <= 0 || L.ntensors <= 0) return cudaSuccess;
    return launch_pdl(adamw_kernel, dim3((unsigned)L.nchunks), dim3(256), 0, s, L);
}

}  // namespace ma
