// Newton-Schulz in fp32 on the CUDA cores (precision mode 1).
//
// The same four steps as the tensor-core path (GRAM, GRAMSQ, APPLY, FINAL;
// see ns_tc.cu), with fp32 operands, fp32 accumulation and fp32 Gram
// buffers. The tf32 tensor-core kind keeps only 10 mantissa bits, too few for
// a 1e-5 match, so this mode uses plain FFMA. It exists for correctness and
// has no performance target. A 64x64 output tile per 256-thread block, a
// 16-deep k slice in shared memory, and 4x4 outputs per thread. The Gram is
// computed in full (no symmetry shortcut).
#include "common.cuh"
#include "internal.h"

namespace ma {

namespace {

constexpr int TS = 64, TK = 16;

template <int MODE>
__global__ void __launch_bounds__(256) ns_simt_kernel(const __grid_constant__ NsParams p, const float* __restrict__ xb,
                                                      const float* __restrict__ gb) {
    __shared__ float As[TK][TS + 4];
    __shared__ float Bs[TK][TS + 4];
    griddep_launch_dependents();
    griddep_wait();
    const int u = blockIdx.z;
    const int i0 = blockIdx.y * TS, j0 = blockIdx.x * TS;
    const bool gram = (MODE == NS_GRAM || MODE == NS_GRAMSQ);
    const int M = p.m;
    const int N = gram ? p.m : p.n;
    const int K = (MODE == NS_GRAM) ? p.n : p.m;
    // operand sources: A(i,k) = SA[i*lda + k]; GRAM-like: B(k,j) = SB[j*ldb + k]; APPLY: B(k,j) = SB[k*ldb + j]
    const float* SA;
    const float* SB;
    int64_t lda, ldb;
    int64_t a_unit, b_unit;  // elements per unit of the operands' buffers (guarded build)
    if (MODE == NS_GRAM) {
        SA = xb + (int64_t)u * p.x_unit; lda = p.ldx; a_unit = p.x_unit;
        SB = SA; ldb = p.ldx; b_unit = p.x_unit;
    } else if (MODE == NS_GRAMSQ) {
        SA = reinterpret_cast<const float*>(p.xin) + (int64_t)u * p.g_unit; lda = p.ldg; a_unit = p.g_unit;
        SB = SA; ldb = p.ldg; b_unit = p.g_unit;
    } else {
        SA = gb + (int64_t)u * p.g_unit; lda = p.ldg; a_unit = p.g_unit;
        SB = xb + (int64_t)u * p.x_unit; ldb = p.ldx; b_unit = p.x_unit;
    }
    // element offsets from the buffers' starts, and their extents
    [[maybe_unused]] const int64_t a0 = (int64_t)u * a_unit, a_ext = (int64_t)p.units * a_unit;
    [[maybe_unused]] const int64_t b0 = (int64_t)u * b_unit, b_ext = (int64_t)p.units * b_unit;
    const int tid = threadIdx.x;
    const int ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += TK) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // A tile: 64 rows x 16 k, k fastest
            const int idx = tid * 4 + e;
            const int ii = idx >> 4, kk = idx & 15;
            const int gi = i0 + ii, gk = k0 + kk;
            As[kk][ii] = (gi < M && gk < K && MA_INB(a0 + (int64_t)gi * lda + gk, 1, a_ext, p.status))
                             ? SA[(int64_t)gi * lda + gk] : 0.f;
        }
        if (gram) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int idx = tid * 4 + e;
                const int jj = idx >> 4, kk = idx & 15;
                const int gj = j0 + jj, gk = k0 + kk;
                Bs[kk][jj] = (gj < N && gk < K && MA_INB(b0 + (int64_t)gj * ldb + gk, 1, b_ext, p.status))
                                 ? SB[(int64_t)gj * ldb + gk] : 0.f;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int idx = tid * 4 + e;
                const int kk = idx >> 6, jj = idx & 63;
                const int gj = j0 + jj, gk = k0 + kk;
                Bs[kk][jj] = (gj < N && gk < K && MA_INB(b0 + (int64_t)gk * ldb + gj, 1, b_ext, p.status))
                                 ? SB[(int64_t)gk * ldb + gj] : 0.f;
            }
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) a[r] = As[kk][ty * 4 + r];
#pragma unroll
            for (int c = 0; c < 4; ++c) b[c] = Bs[kk][tx * 4 + c];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
        }
        __syncthreads();
    }
    const float sa = (p.first && p.scale) ? p.scale[u] : 1.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = i0 + ty * 4 + r;
        if (i >= M) continue;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int j = j0 + tx * 4 + c;
            if (j >= N) continue;
            const float v = acc[r][c];
            const int64_t gi = (int64_t)u * p.g_unit + (int64_t)i * p.ldg + j;  // (i, j) in a Gram buffer
            const int64_t xi = (int64_t)u * p.x_unit + (int64_t)i * p.ldx + j;  // (i, j) in an X buffer
            [[maybe_unused]] const int64_t g_ext = (int64_t)p.units * p.g_unit;
            [[maybe_unused]] const int64_t x_ext = (int64_t)p.units * p.x_unit;
            if (MODE == NS_GRAM) {
                float coef = p.coef_gram;
                if (p.first) coef *= sa * sa;
                if (MA_INB(gi, 1, g_ext, p.status)) reinterpret_cast<float*>(p.out)[gi] = coef * v;
            } else if (MODE == NS_GRAMSQ) {
                if (!MA_INB(gi, 1, g_ext, p.status)) continue;
                const float ain = SA[(int64_t)i * lda + j];
                reinterpret_cast<float*>(p.out)[gi] = p.b * ain + p.c * v;
            } else {
                if (!MA_INB(xi, 1, x_ext, p.status)) continue;
                const float x = xb[xi];
                const float o = sa * (p.a * x + v);
                if (MODE == NS_APPLY) {
                    reinterpret_cast<float*>(p.out)[xi] = o;
                } else {
                    const int bidx = u / p.heads, h = u - bidx * p.heads;
                    const int64_t wi = (int64_t)h * p.Rh * p.C + (p.transposed ? (int64_t)j * p.C + i : (int64_t)i * p.C + j);
                    if (!MA_INB(wi, 1, (int64_t)p.heads * p.Rh * p.C, p.status)) continue;
                    float* w = p.W[bidx] + wi;
                    const float wv = *w;
                    *w = p.cautious ? (o * wv > 0.f ? wv - p.lr_wd * wv : wv) - p.lr_s * o : wv * p.decay - p.lr_s * o;
                }
            }
        }
    }
}

}  // namespace

cudaError_t launch_ns_simt(int mode, const NsParams& p, const void* x_buf, const void* g_buf, cudaStream_t s) {
    const bool gram = (mode == NS_GRAM || mode == NS_GRAMSQ);
    const int N = gram ? p.m : p.n;
    dim3 grid((N + TS - 1) / TS, (p.m + TS - 1) / TS, p.units);
    if (p.units == 0 || p.m == 0 || N == 0) return cudaSuccess;
    const float* xb = reinterpret_cast<const float*>(x_buf);
    const float* gb = reinterpret_cast<const float*>(g_buf);
    switch (mode) {
        case NS_GRAM: return launch_pdl(ns_simt_kernel<NS_GRAM>, grid, dim3(256), 0, s, p, xb, gb);
        case NS_GRAMSQ: return launch_pdl(ns_simt_kernel<NS_GRAMSQ>, grid, dim3(256), 0, s, p, xb, gb);
        case NS_APPLY: return launch_pdl(ns_simt_kernel<NS_APPLY>, grid, dim3(256), 0, s, p, xb, gb);
        case NS_FINAL: return launch_pdl(ns_simt_kernel<NS_FINAL>, grid, dim3(256), 0, s, p, xb, gb);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ma
