// Launch descriptors shared between the host entry points (api.cu) and the
// kernel files. Every table a kernel needs travels in its parameter block
// (up to 32 KB on sm_70+ with CUDA >= 12.1), so no call allocates device
// memory and every launch can be replayed from a CUDA graph as captured.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/muonadamw.h"

namespace ma {

// ------------------------------------------------------------------ per-device host caches

constexpr int kMaxDevices = 64;

// A value looked up once per device (a symbol address, an occupancy figure,
// kernel attributes set), safe when several host threads make their first
// call on a device at the same time: the lookup runs under a mutex, at most
// once per device while it succeeds, and readers after that take no lock.
// A failed lookup is not cached, so the next call tries again. Objects of
// this type live in static storage (zero-initialised before any call).
template <typename T>
class PerDevice {
  public:
    // *out = the cached value of device `dev`, computed by init(&value) (which
    // returns a cudaError_t) on the first successful call.
    template <typename Init>
    cudaError_t get(int dev, T* out, Init init) {
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        if (!ready_[dev].load(std::memory_order_acquire)) {
            std::lock_guard<std::mutex> lock(mu_);
            if (!ready_[dev].load(std::memory_order_relaxed)) {
                T v{};
                const cudaError_t e = init(&v);
                if (e != cudaSuccess) return e;
                val_[dev] = v;
                ready_[dev].store(1, std::memory_order_release);
            }
        }
        *out = val_[dev];
        return cudaSuccess;
    }

  private:
    std::mutex mu_;
    std::atomic<int> ready_[kMaxDevices];
    T val_[kMaxDevices];
};

// ------------------------------------------------------------------ AdamW

constexpr int kAdamwChunk = 8192;              // elements per block
constexpr int kAdamwMaxTensorsPerLaunch = 320;  // parameter-block capacity

struct AdamwTensorDesc {
    float* p;
    const void* g;
    float* m;
    float* v;
    int64_t numel;
    int64_t chunk0;  // first global chunk index of this tensor
    int32_t group;
    int32_t vec;     // 1 when p, m, v are 16-byte aligned and g is aligned for 4-wide loads
};

struct AdamwGroupConst {
    float decay;         // 1 - lr * wd
    float step_size;     // lr / (1 - beta1^t)
    float inv_sqrt_bc2;  // 1 / sqrt(1 - beta2^t)
    float beta1, beta2, omb1, omb2, eps;
};

struct AdamwLaunch {
    int32_t ntensors;
    int32_t gdt;  // ma_dtype_t of every gradient in this launch
    int64_t nchunks;
    int* status;  // device status word (guarded indexing in debug builds)
    AdamwGroupConst grp[MA_MAX_GROUPS];
    AdamwTensorDesc t[kAdamwMaxTensorsPerLaunch];
};

cudaError_t launch_adamw(const AdamwLaunch& L, cudaStream_t s);
const void* adamw_kernel_func();  // the kernel's host-side handle (CUDA-graph node matching)

// ------------------------------------------------------------------ Muon: momentum + norm

constexpr int kPrepChunk = 8192;      // elements per chunk (one partial sum each), flat path
constexpr int kPrepSideThreads = 128;  // threads per block of the side-stream flat kernel
constexpr int kPrepTRows = 64;        // transposing path: rows of u per thread block (16 per warp)
constexpr int kPrepTCols = 64;        // transposing path: columns of u per thread block (2 per lane)

struct MuonPrepLaunch {
    int32_t batch, heads, transposed, gdt, nesterov, x_f32;
    int* status;          // device status word (guarded indexing in debug builds)
    int64_t C, Rh;        // matrix columns, rows per head slice
    int64_t ldx;          // row stride (elements) of the NS operand X
    int64_t x_unit;       // elements between consecutive units of X
    int64_t parts;        // partial sums per unit
    int64_t tiles_c;      // transposing path: blocks of kPrepTCols columns along C
    float beta, omb;
    void* X;
    double* partials;
    const void* G[MA_MAX_BATCH];
    float* M[MA_MAX_BATCH];
};

// Number of per-block partial sums the momentum pass writes for one unit.
int64_t prep_parts_per_unit(int64_t Rh, int64_t C, int transposed);

// max_blocks > 0: at most that many blocks (a small grid that runs beside the
// Newton-Schulz kernels of another batch, with the same partial sums; the
// flat path then takes its side-stream kernel); 0: one block per chunk.
cudaError_t launch_muon_prep(const MuonPrepLaunch& L, int max_blocks, cudaStream_t s);
// Per-device kernel attributes of the momentum kernels, ahead of a stream capture.
cudaError_t prep_setup();
// scale[u] = 1 / (sqrt(sum of the unit's partials) + eps), deterministic order.
cudaError_t launch_norm_finalize(const double* partials, int64_t parts, int units, float eps, float* scale,
                                 cudaStream_t s);

// ------------------------------------------------------------------ Newton-Schulz

enum NsMode { NS_GRAM = 0, NS_APPLY = 1, NS_FINAL = 2, NS_GRAMSQ = 3 };


struct NsParams {
    int32_t units, m, n;
    int64_t ldx, ldg;        // row strides (elements) of X and of the Gram
    int64_t x_unit, g_unit;  // elements between consecutive units
    int32_t first;           // 1: fold the per-unit normalisation scale in
    float a, b, c;           // this iteration's polynomial coefficients
    float coef_gram;         // GRAM epilogue multiplier (b, or 1 when c != 0)
    const float* scale;      // per-unit 1 / (||u|| + eps); may be NULL when first == 0
    const void* xin;         // APPLY/FINAL: X of this iteration; GRAMSQ: the Gram input A
    const void* zin;         // GRAMSQ: second operand Z, symmetric and commuting with A (NULL: A itself);
                             // the launch computes b*Z + c*(A Z) on the upper tiles and mirrors them
    void* out;               // GRAM/GRAMSQ: Gram output; APPLY: next X
    // FINAL: W <- W * decay - lr_s * X_N, written through W[] in the original orientation
    int32_t transposed, heads;
    int64_t Rh, C;
    float decay, lr_s;
    float lr_wd;             // lr * wd, for cautious decay
    int32_t cautious;        // decay only where X_N * W > 0
    long long wait_limit_ns;
    int* status;             // per-device status word
    float* W[MA_MAX_BATCH];
};

// bf16 tcgen05 path: X, Gram buffers are bf16 with 16-byte-multiple strides.
size_t ns_tc_smem_bytes();
cudaError_t launch_ns_tc(int mode, const NsParams& p, const void* x_buf, const void* g_buf, int num_sms,
                         cudaStream_t s);
// Several jobs (same mode) in one persistent launch: at most ns_tc_max_jobs()
// jobs and, for the final apply, ns_tc_max_weights() weight matrices in total.
struct NsJobIn {
    const NsParams* p;
    const void* x_buf;
    const void* g_buf;
};
// *launched (may be null) is increased by the number of kernels launched: one
// for jobs with m > 128, one for jobs with m <= 128 (single-CTA tiles).
cudaError_t launch_ns_tc_group(int mode, const NsJobIn* jobs, int njobs, int num_sms, cudaStream_t s,
                               int* launched);
int ns_tc_max_jobs();
int ns_tc_max_weights();
// Per-device kernel attributes of every instance, ahead of a stream capture.
cudaError_t ns_tc_setup(int num_sms);
// CUDA-graph support: whether a kernel node's function is a final apply, the
// size of its single (by value) parameter, and an in-place update of the
// decay terms of each of its jobs. f(ctx, first weight of the job, rows per
// unit, columns, &decay, &lr_s, &lr_wd) returns nonzero to stop with that code.
typedef int (*NsFinalPatchFn)(void* ctx, const float* W, int64_t Rh, int64_t C, float* decay, float* lr_s,
                              float* lr_wd);
bool ns_tc_is_final(const void* func);
size_t ns_tc_launch_bytes();
int ns_tc_patch_final(void* launch, NsFinalPatchFn f, void* ctx);

// Q = a*I + b*A (bf16 m x m per unit, row stride ldg, unit stride g_unit).
// status: the device status word (guarded indexing in debug builds).
cudaError_t launch_ns_q1(const void* A, void* Q, int m, int64_t ldg, int64_t g_unit, int units, float a, float b,
                         int* status, int num_sms, cudaStream_t s);

// fp32 SIMT path (precision mode 1).
cudaError_t launch_ns_simt(int mode, const NsParams& p, const void* x_buf, const void* g_buf, cudaStream_t s);

// ------------------------------------------------------------------ misc

cudaError_t launch_wait_selftest(long long limit_ns, int* status, cudaStream_t s);
long long host_wait_limit_ns();
int* device_status_ptr();  // address of this device's status word, NULL on failure

}  // namespace ma
