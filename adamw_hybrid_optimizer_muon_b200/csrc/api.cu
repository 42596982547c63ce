// C ABI of the MuonAdamW library: validation, workspace layout, the per-step
// orchestration of the kernels, and the plan over a parameter table.
//
// Structure of one step ("How nanochat Combines Muon and AdamW in a Single
// Optimizer", "The MuonAdamW Class Architecture": one step() that dispatches
// on each group's kind):
//   1. one multi-tensor AdamW launch over every AdamW tensor (adamw.cu)
//   2. per Muon sub-batch of same-shape matrices ("Muon Step Implementation":
//      stacked batches): momentum + norm (muon_prep.cu) and the norm
//      finalize, then the Newton-Schulz chain (ns_tc.cu, or ns_simt.cu in
//      fp32 mode), whose last GEMM writes the decayed, updated weights.
//      Consecutive sub-batches whose chains take the same kernels share each
//      Newton-Schulz launch.
// The plan splits buckets into sub-batches (workspace within the caller's cap,
// or 4 GiB), groups small ones, and can replay the whole step from a CUDA
// graph. The host never synchronises. Every argument is checked before the
// first launch, so a failing call changes nothing.
#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <unordered_map>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

namespace ma {

__device__ int g_status = 0;

static std::atomic<long long> g_host_wait_limit_ns{2000000000LL};
// Plans created while this is set get two workspace halves and run momentum
// passes on a side stream (ma_set_momentum_overlap).
static std::atomic<int> g_momentum_overlap{0};
long long host_wait_limit_ns() { return g_host_wait_limit_ns.load(std::memory_order_relaxed); }

int* device_status_ptr() {
    static PerDevice<int*> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    int* ptr = nullptr;
    const cudaError_t e = cache.get(dev, &ptr, [](int** v) {
        void* p = nullptr;
        const cudaError_t r = cudaGetSymbolAddress(&p, g_status);
        *v = reinterpret_cast<int*>(p);
        return r;
    });
    return e == cudaSuccess ? ptr : nullptr;
}

namespace {

// ------------------------------------------------------------------ launch profiler

struct ProfRec {
    int ev;  // index of the event pair in the pool
    int cls;
    double flops, bytes;
};
thread_local bool g_prof_on = false;
thread_local std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_prof_pool;
thread_local std::vector<ProfRec> g_prof_recs;

// Returns the record index, or -1 when profiling is off or an event is unavailable.
int prof_begin(int cls, cudaStream_t s) {
    if (!g_prof_on) return -1;
    const size_t k = g_prof_recs.size();
    if (k >= g_prof_pool.size()) {
        cudaEvent_t a, b;
        if (cudaEventCreate(&a) != cudaSuccess) return -1;
        if (cudaEventCreate(&b) != cudaSuccess) {
            cudaEventDestroy(a);
            return -1;
        }
        g_prof_pool.push_back({a, b});
    }
    if (cudaEventRecord(g_prof_pool[k].first, s) != cudaSuccess) return -1;
    g_prof_recs.push_back({(int)k, cls, 0.0, 0.0});
    return (int)k;
}

void prof_end(int rec, cudaStream_t s, double flops, double bytes) {
    if (rec < 0) return;
    ProfRec& r = g_prof_recs[rec];
    r.flops = flops;
    r.bytes = bytes;
    cudaEventRecord(g_prof_pool[r.ev].second, s);
}

constexpr size_t kAlign = 256;
// Muon sub-batch sizes when gradients stream in from the host: the first
// sub-batch is small so that compute starts after a short copy, the others
// large enough to keep every GEMM launch many waves deep.
constexpr int kFromHostFirstBatch = 2;
constexpr int kFromHostBatch = 32;
// Workspace that a plan may use, beyond its largest sub-batch, to run small
// Muon buckets through shared Newton-Schulz launches.
constexpr size_t kGroupWsBytes = size_t(4) << 30;
// Without a cap from the caller, a bucket's sub-batches are halved until their
// workspace is at most this. Fewer units per launch keep the pairs of a
// launch on a narrower band of units, so more operand tiles are still in L2
// when the next wave reads them: on the 7B set, sub-batches of 32 and 16
// matrices took 333 ms a step against 342-350 ms for whole buckets, with a
// quarter of the workspace.
constexpr size_t kSubBatchBytes = size_t(4) << 30;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t round8(int64_t x) { return (x + 7) / 8 * 8; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// sm_100a code runs only on compute capability 10.0; cache per device.
int device_ok_and_sms(int* sms) {
    // per device: the SM count, or -MA_ERR_* when the device cannot run this library
    static PerDevice<int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MA_ERR_UNSUPPORTED;
    int v = 0;
    const cudaError_t e = cache.get(dev, &v, [dev](int* out) {
        int maj = 0, min = 0, n = 0, smem = 0;
        if (cudaDeviceGetAttribute(&maj, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&min, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return cudaErrorUnknown;  // not cached: the next call asks again
        if (maj != 10 || min != 0 || (size_t)smem < ns_tc_smem_bytes() || n < 2) *out = -MA_ERR_UNSUPPORTED;
        else *out = n;
        return cudaSuccess;
    });
    if (e != cudaSuccess) return MA_ERR_CUDA;
    if (v < 0) return -v;
    if (sms) *sms = v;
    return MA_OK;
}

// ------------------------------------------------------------------ Muon geometry

struct MuonGeom {
    int64_t R, C, Rh;
    int heads, transposed;
    int64_t m, n, ldx, ldg;
    int64_t units;
    int64_t parts;
    int esz;
    bool quintic;
    bool gspace;  // the chain runs in Gram space (gram_space below)
    // standard chain: X0, X1 (ping-pong), Gram, Gram2 (c != 0); Gram-space
    // chain: X0, and four m x m buffers A0 (off_g), A1 (off_g2), Q0, Q1
    size_t off_x0, off_x1, off_g, off_g2, off_q0, off_q1, off_part, off_scale, total;
};

bool any_c(const ma_muon_hparams_t& hp) {
    const int nc = hp.n_coeffs;
    for (int k = 0; k < nc && k < MA_MAX_NS_STEPS; ++k)
        if (hp.coeffs[k][2] != 0.f) return true;
    return false;
}

int check_muon_hp(const ma_muon_hparams_t* hp) {
    if (!hp) return MA_ERR_NULL;
    if (hp->ns_steps < 1 || hp->ns_steps > MA_MAX_NS_STEPS) return MA_ERR_ARG;
    if (!(hp->n_coeffs == 1 || hp->n_coeffs == hp->ns_steps)) return MA_ERR_ARG;
    if (hp->scale_mode < 0 || hp->scale_mode > 2) return MA_ERR_ARG;
    if (hp->precision < 0 || hp->precision > 1) return MA_ERR_ARG;
    if (hp->heads < 1) return MA_ERR_SHAPE;
    if (!(hp->beta >= 0.f && hp->beta <= 1.f)) return MA_ERR_ARG;
    if (!(hp->eps >= 0.f) || !std::isfinite(hp->lr) || !std::isfinite(hp->weight_decay)) return MA_ERR_ARG;
    for (int k = 0; k < hp->n_coeffs; ++k)
        for (int j = 0; j < 3; ++j)
            if (!std::isfinite(hp->coeffs[k][j])) return MA_ERR_ARG;
    return MA_OK;
}

// Whether a unit's Newton-Schulz chain runs in Gram space. The iteration
// X_{k+1} = P_k X_k, P_k = a_k I + b_k A_k, A_k = X_k X_k^T, gives
// X_N = Q_N X_0 with Q_N = P_{N-1} ... P_0, and A_{k+1} = P_k A_k P_k: every
// factor is a polynomial in A_0, so all of them are symmetric and commute.
// The chain then forms A_0 (one Gram, m(m+1)n flops), updates Q, A and
// Y = A P with symmetric m x m products (m(m+1)m flops each, 3N - 3 of them)
// and applies Q_N to X_0 once (2m^2 n): for N = 5 and n = 2.69 m (the 7B
// set's MLP matrices, or 128 x 4096 head slices) a fraction of the flops of
// N Grams and N applies. Taken for bf16 operands without an A^2 term when
// n >= 1.25 m, m >= 128 and m n >= 2^19 (on smaller units the 3N + 1
// launches cost more than the flops saved); exact in real arithmetic, and
// within the same bf16 error as the direct iteration.
bool gram_space(int64_t m, int64_t n, const ma_muon_hparams_t& hp) {
    return hp.precision == 0 && !any_c(hp) && m >= 128 && 4 * n >= 5 * m && m * n >= (int64_t(1) << 19);
}

int muon_geom(int batch, int64_t R, int64_t C, const ma_muon_hparams_t& hp, MuonGeom* g) {
    if (batch < 0 || R < 0 || C < 0) return MA_ERR_SHAPE;
    if (hp.heads < 1 || (R > 0 && R % hp.heads != 0)) return MA_ERR_SHAPE;
    g->R = R;
    g->C = C;
    g->heads = hp.heads;
    g->Rh = R / hp.heads;
    g->transposed = g->Rh > C ? 1 : 0;
    g->m = std::min(g->Rh, C);
    g->n = std::max(g->Rh, C);
    g->ldx = round8(g->n);
    g->ldg = round8(g->m);
    g->units = (int64_t)batch * hp.heads;
    g->parts = (g->Rh > 0 && C > 0) ? prep_parts_per_unit(g->Rh, C, g->transposed) : 0;
    g->esz = hp.precision ? 4 : 2;
    g->quintic = any_c(hp);
    g->gspace = gram_space(g->m, g->n, hp);
    size_t off = 0;
    const size_t xbytes = (size_t)g->units * g->m * g->ldx * g->esz;
    const size_t gbytes = (size_t)g->units * g->m * g->ldg * g->esz;
    g->off_x0 = off;
    off = align_up(off + xbytes, kAlign);
    if (!g->gspace) {
        g->off_x1 = off;
        if (hp.ns_steps >= 2) off = align_up(off + xbytes, kAlign);
        g->off_g = off;
        off = align_up(off + gbytes, kAlign);
        g->off_g2 = off;
        if (g->quintic) off = align_up(off + gbytes, kAlign);
        g->off_q0 = g->off_q1 = off;  // unused
    } else {
        g->off_x1 = g->off_x0;  // unused
        g->off_g = off;
        off = align_up(off + gbytes, kAlign);
        g->off_g2 = off;
        off = align_up(off + gbytes, kAlign);
        g->off_q0 = off;
        off = align_up(off + gbytes, kAlign);
        g->off_q1 = off;
        off = align_up(off + gbytes, kAlign);
    }
    g->off_part = off;
    off = align_up(off + (size_t)g->units * g->parts * sizeof(double), kAlign);
    g->off_scale = off;
    off = align_up(off + (size_t)g->units * sizeof(float), kAlign);
    g->total = (batch == 0 || R == 0 || C == 0) ? 0 : off;
    return MA_OK;
}

float shape_scale(int64_t R, int64_t C, int mode) {
    const double r = (double)R / (double)C;
    if (mode == 0) return (float)std::sqrt(std::max(1.0, r));
    if (mode == 1) return (float)std::sqrt(r);
    return 1.f;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MA_OK : MA_ERR_CUDA; }

int ns_prof_class(int mode) {
    return mode == NS_GRAM     ? MA_PROF_NS_GRAM
           : mode == NS_GRAMSQ ? MA_PROF_NS_GRAMSQ
           : mode == NS_FINAL  ? MA_PROF_NS_FINAL
                               : MA_PROF_NS_APPLY;
}

// Algorithmic flops of one Newton-Schulz launch. A symmetric Gram X X^T has
// m(m+1)/2 distinct entries of n multiply-adds each: m(m+1)n flops (A A^T:
// m(m+1)m). The apply B X costs 2 m^2 n.
double ns_flops(int mode, int64_t units, int64_t m, int64_t n) {
    const double u = (double)units, M = (double)m, N = (double)n;
    if (mode == NS_GRAM) return u * M * (M + 1.0) * N;
    if (mode == NS_GRAMSQ) return u * M * (M + 1.0) * M;
    return u * 2.0 * M * M * N;
}

// One Muon batch of same-shape matrices with its own workspace (g.total bytes).
struct MuonJob {
    int batch;
    MuonGeom g;
    float* const* W;
    const void* const* G;
    int gdt;
    float* const* M;
    const ma_muon_hparams_t* hp;
    uint8_t* ws;
};

// Bit k set: Newton-Schulz iteration k has c != 0 (it needs the A^2 term).
uint32_t quint_mask(const ma_muon_hparams_t& hp) {
    uint32_t mask = 0;
    for (int k = 0; k < hp.ns_steps && k < MA_MAX_NS_STEPS; ++k)
        if (hp.coeffs[hp.n_coeffs == 1 ? 0 : k][2] != 0.f) mask |= 1u << k;
    return mask;
}

// Jobs can share Newton-Schulz launches when they take the same sequence of
// kernels: the tensor-core path, the same number of iterations and the same
// iterations with an A^2 term. Coefficients, learning rates and decay may differ.
bool ns_compatible(const ma_muon_hparams_t& x, const ma_muon_hparams_t& y) {
    return x.precision == 0 && y.precision == 0 && x.ns_steps == y.ns_steps && quint_mask(x) == quint_mask(y);
}

// Momentum + norm partials, then the norm finalize, of one job.
int muon_prep(const MuonJob& j, cudaStream_t s, int max_blocks, bool side, int* launches) {
    const MuonGeom& g = j.g;
    const ma_muon_hparams_t& hp = *j.hp;
    double* part = reinterpret_cast<double*>(j.ws + g.off_part);
    float* scale = reinterpret_cast<float*>(j.ws + g.off_scale);
    MuonPrepLaunch P;
    std::memset(&P, 0, sizeof(P));
    P.batch = j.batch;
    P.status = device_status_ptr();
    P.heads = g.heads;
    P.transposed = g.transposed;
    P.gdt = j.gdt;
    P.nesterov = hp.nesterov ? 1 : 0;
    P.x_f32 = hp.precision ? 1 : 0;
    P.C = g.C;
    P.Rh = g.Rh;
    P.ldx = g.ldx;
    P.x_unit = g.m * g.ldx;
    P.parts = g.parts;
    P.tiles_c = (g.C + kPrepTCols - 1) / kPrepTCols;
    P.beta = hp.beta;
    P.omb = 1.f - hp.beta;
    P.X = j.ws + g.off_x0;
    P.partials = part;
    for (int b = 0; b < j.batch; ++b) {
        P.G[b] = j.G[b];
        P.M[b] = j.M[b];
    }
    const double elems = (double)g.units * (double)g.Rh * (double)g.C;
    int pr = prof_begin(side ? MA_PROF_MOMENTUM_SIDE : MA_PROF_MOMENTUM, s);
    int st = cuda_status(launch_muon_prep(P, max_blocks, s));
    prof_end(pr, s, 0.0, elems * ((j.gdt == MA_BF16 ? 2 : 4) + 8 + (hp.precision ? 4 : 2)));
    if (st) return st;
    // on the side stream the finalize shares the SMs with the chain before it, like the pass
    pr = prof_begin(side ? MA_PROF_MOMENTUM_SIDE : MA_PROF_FINALIZE, s);
    st = cuda_status(launch_norm_finalize(part, g.parts, (int)g.units, hp.eps, scale, s));
    prof_end(pr, s, 0.0, (double)g.units * g.parts * 8.0 + g.units * 4.0);
    if (st) return st;
    *launches += 2;
    return MA_OK;
}

// Algorithmic DRAM bytes of one Newton-Schulz launch: each operand read once
// and each result written once (esz bytes per element: 2 for bf16, 4 in fp32
// mode). The final apply also reads and writes the fp32 weights.
double ns_bytes(int mode, int64_t units, int64_t m, int64_t n, int esz) {
    const double u = (double)units, M = (double)m, N = (double)n, e = (double)esz;
    if (mode == NS_GRAM) return u * e * (M * N + M * M);
    if (mode == NS_GRAMSQ) return u * e * 3.0 * M * M;  // A and Z read, the product written
    if (mode == NS_APPLY) return u * e * (M * M + 2.0 * M * N);
    return u * (e * (M * M + M * N) + 8.0 * M * N);
}

// All checks passed; launch the whole Muon chain for a set of jobs that are
// pairwise ns_compatible (or a single job). Each Newton-Schulz step is one
// launch over every job's tiles on the tensor-core path; per job in fp32 mode.
// A tile's arithmetic does not depend on the launch it is in, so grouping
// gives the same bits as running the jobs one by one.
// The momentum passes (and norm finalizes) of a set of jobs. max_blocks > 0
// bounds the flat momentum kernel's grid (see launch_muon_prep).
int prep_jobs(const MuonJob* jobs, int njobs, cudaStream_t s, int max_blocks, int* launches, bool side = false) {
    int st;
    for (int j = 0; j < njobs; ++j)
        if (jobs[j].g.total > 0 && (st = muon_prep(jobs[j], s, max_blocks, side, launches))) return st;
    return MA_OK;
}

// Newton-Schulz parameters of a job that do not change along its chain:
// geometry, the normalisation scales, the final decay and update.
NsParams base_params(const MuonJob& J) {
    const MuonGeom& g = J.g;
    const ma_muon_hparams_t& hp = *J.hp;
    NsParams q;
    std::memset(&q, 0, sizeof(q));
    q.units = (int)g.units;
    q.m = (int)g.m;
    q.n = (int)g.n;
    q.ldx = g.ldx;
    q.ldg = g.ldg;
    q.x_unit = g.m * g.ldx;
    q.g_unit = g.m * g.ldg;
    q.scale = reinterpret_cast<float*>(J.ws + g.off_scale);
    q.transposed = g.transposed;
    q.heads = g.heads;
    q.Rh = g.Rh;
    q.C = g.C;
    q.decay = 1.f - hp.lr * hp.weight_decay;
    q.lr_s = hp.lr * shape_scale(g.Rh, g.C, hp.scale_mode);
    q.lr_wd = hp.lr * hp.weight_decay;
    q.cautious = hp.cautious ? 1 : 0;
    q.wait_limit_ns = host_wait_limit_ns();
    q.status = device_status_ptr();
    for (int b = 0; b < J.batch; ++b) q.W[b] = J.W[b];
    return q;
}

// The Gram-space chain (gram_space) of a set of jobs, the launches shared:
//   A_0 = s^2 X_0 X_0^T                       (Gram, into A)
//   Q_1 = a_0 I + b_0 A_0                     (elementwise)
//   per iteration k: Q_{k+1} = a_k Q_k + b_k A_k Q_k   (k >= 1)
//                    Y = a_k A_k + b_k A_k A_k, A_{k+1} = a_k Y + b_k A_k Y   (k < N - 1)
//   W <- W (1 - lr wd) - lr scale (s Q_N X_0)  (final apply)
// Each m x m product is symmetric (all factors are polynomials in A_0): the
// symmetric-product launches compute its upper tiles and mirror them. Y goes
// to the Q buffer that the Q update has just freed, so four m x m buffers do.
int chain_gspace(const std::vector<const MuonJob*>& jobs, cudaStream_t s, int sms, int* launches) {
    const int nj = (int)jobs.size();
    if (nj == 0) return MA_OK;
    if (nj > ns_tc_max_jobs()) return MA_ERR_UNSUPPORTED;
    const int steps = jobs[0]->hp->ns_steps;  // the same for every job of the set
    std::vector<NsParams> p(nj);
    std::vector<void*> X0(nj), Acur(nj), Anext(nj), Qcur(nj), Qfree(nj);
    for (int i = 0; i < nj; ++i) {
        const MuonJob& J = *jobs[i];
        p[i] = base_params(J);
        X0[i] = J.ws + J.g.off_x0;
        Acur[i] = J.ws + J.g.off_g;
        Anext[i] = J.ws + J.g.off_g2;
        Qcur[i] = J.ws + J.g.off_q0;
        Qfree[i] = J.ws + J.g.off_q1;
    }
    std::vector<NsJobIn> in(nj);
    // one launch over every job; xb: the X operand (Gram and final apply), gb: the m x m operand
    auto launch = [&](int mode, const std::vector<void*>& xb, const std::vector<void*>& gb) -> int {
        const int pr = prof_begin(ns_prof_class(mode), s);
        double flops = 0.0, bytes = 0.0;
        for (int i = 0; i < nj; ++i) {
            in[i] = {&p[i], xb[i], gb[i]};
            const MuonGeom& g = jobs[i]->g;
            flops += ns_flops(mode, g.units, g.m, g.n);
            bytes += ns_bytes(mode, g.units, g.m, g.n, g.esz);
        }
        const cudaError_t e = launch_ns_tc_group(mode, in.data(), nj, sms, s, launches);
        prof_end(pr, s, flops, bytes);
        return cuda_status(e);
    };
    auto coef = [&](int i, int k, int which) {
        const ma_muon_hparams_t& hp = *jobs[i]->hp;
        return hp.coeffs[hp.n_coeffs == 1 ? 0 : k][which];
    };
    int st;
    // A_0, normalised: the Gram with multiplier 1 (times s^2 on the first iteration)
    for (int i = 0; i < nj; ++i) {
        p[i].first = 1;
        p[i].coef_gram = 1.f;
        p[i].out = Acur[i];
    }
    if ((st = launch(NS_GRAM, X0, Acur))) return st;
    for (int i = 0; i < nj; ++i) {
        const MuonGeom& g = jobs[i]->g;
        const int pr = prof_begin(MA_PROF_NS_Q1, s);
        const cudaError_t e = launch_ns_q1(Acur[i], Qcur[i], (int)g.m, g.ldg, g.m * g.ldg, (int)g.units,
                                           coef(i, 0, 0), coef(i, 0, 1), device_status_ptr(), sms, s);
        prof_end(pr, s, 0.0, 4.0 * (double)g.units * (double)g.m * (double)g.m);  // A read, Q written (bf16)
        if (e != cudaSuccess) return MA_ERR_CUDA;
        ++*launches;
    }
    // a symmetric product out = alpha Z + beta A Z over every job (Z = A when z is null)
    auto symprod = [&](const std::vector<void*>& A, const std::vector<void*>* Z, const std::vector<void*>& out,
                       int k) -> int {
        for (int i = 0; i < nj; ++i) {
            p[i].first = 0;
            p[i].xin = A[i];
            p[i].zin = Z ? (*Z)[i] : nullptr;
            p[i].out = out[i];
            p[i].b = coef(i, k, 0);
            p[i].c = coef(i, k, 1);
        }
        return launch(NS_GRAMSQ, X0, A);
    };
    for (int k = 0; k < steps; ++k) {
        if (k >= 1) {
            if ((st = symprod(Acur, &Qcur, Qfree, k))) return st;  // Q_{k+1}
            std::swap(Qcur, Qfree);                                  // Qfree: Q_k, no longer needed
        }
        if (k + 1 < steps) {
            if ((st = symprod(Acur, nullptr, Qfree, k))) return st;  // Y = A P, in the free Q buffer
            if ((st = symprod(Acur, &Qfree, Anext, k))) return st;   // A_{k+1} = P Y
            std::swap(Acur, Anext);
        }
    }
    // X_N = s Q_N X_0, written into W by the final apply (a = 0: no a X term)
    for (int i = 0; i < nj; ++i) {
        p[i].first = 1;
        p[i].a = 0.f;
        p[i].b = 1.f;
        p[i].c = 0.f;
        p[i].zin = nullptr;
        p[i].xin = X0[i];
        p[i].out = nullptr;
    }
    return launch(NS_FINAL, X0, Qcur);
}

// The Newton-Schulz chain of a set of jobs whose momentum passes are done:
// the Gram-space chain where it pays (gram_space), the direct iteration for
// the rest.
int chain_jobs(const MuonJob* jobs_in, int njobs_in, cudaStream_t s, int sms, int* launches) {
    std::vector<const MuonJob*> jobs, gjobs;
    int st;
    for (int j = 0; j < njobs_in; ++j) {
        if (jobs_in[j].g.total == 0) continue;
        if (jobs_in[j].g.gspace) gjobs.push_back(&jobs_in[j]);
        else jobs.push_back(&jobs_in[j]);
    }
    if ((st = chain_gspace(gjobs, s, sms, launches))) return st;
    const int nj = (int)jobs.size();
    if (nj == 0) return MA_OK;
    if (nj > ns_tc_max_jobs()) return MA_ERR_UNSUPPORTED;

    const ma_muon_hparams_t& hp0 = *jobs[0]->hp;
    std::vector<NsParams> p(nj);
    std::vector<void*> cur(nj), nxt(nj), Gb(nj), G2(nj);
    for (int i = 0; i < nj; ++i) {
        const MuonJob& J = *jobs[i];
        const MuonGeom& g = J.g;
        p[i] = base_params(J);
        cur[i] = J.ws + g.off_x0;
        nxt[i] = J.ws + g.off_x1;
        Gb[i] = J.ws + g.off_g;
        G2[i] = J.ws + g.off_g2;
    }

    std::vector<NsJobIn> in(nj);
    auto launch = [&](int mode, const std::vector<void*>& xb, const std::vector<void*>& gb) -> int {
        const int pr = prof_begin(ns_prof_class(mode), s);
        double flops = 0.0, bytes = 0.0;
        cudaError_t e = cudaSuccess;
        for (int i = 0; i < nj; ++i) {
            in[i] = {&p[i], xb[i], gb[i]};
            const MuonGeom& g = jobs[i]->g;
            flops += ns_flops(mode, g.units, g.m, g.n);
            bytes += ns_bytes(mode, g.units, g.m, g.n, g.esz);
        }
        if (hp0.precision) {
            for (int i = 0; i < nj && e == cudaSuccess; ++i) {
                e = launch_ns_simt(mode, p[i], xb[i], gb[i], s);
                ++*launches;
            }
        } else {
            e = launch_ns_tc_group(mode, in.data(), nj, sms, s, launches);
        }
        prof_end(pr, s, flops, bytes);
        return cuda_status(e);
    };

    for (int k = 0; k < hp0.ns_steps; ++k) {
        bool quint = false;
        for (int i = 0; i < nj; ++i) {
            const ma_muon_hparams_t& hp = *jobs[i]->hp;
            const float* cf = hp.coeffs[hp.n_coeffs == 1 ? 0 : k];
            NsParams& q = p[i];
            q.a = cf[0];
            q.b = cf[1];
            q.c = cf[2];
            q.first = (k == 0) ? 1 : 0;
            quint = cf[2] != 0.f;  // the same for every job of the set
            q.coef_gram = quint ? 1.f : cf[1];
            q.out = Gb[i];
        }
        if ((st = launch(NS_GRAM, cur, Gb))) return st;
        std::vector<void*>* Bbuf = &Gb;
        if (quint) {
            for (int i = 0; i < nj; ++i) {
                p[i].xin = Gb[i];
                p[i].out = G2[i];
            }
            if ((st = launch(NS_GRAMSQ, cur, Gb))) return st;
            Bbuf = &G2;
        }
        const bool last = k + 1 == hp0.ns_steps;
        for (int i = 0; i < nj; ++i) {
            p[i].xin = cur[i];
            p[i].out = last ? nullptr : nxt[i];
        }
        if ((st = launch(last ? NS_FINAL : NS_APPLY, cur, *Bbuf))) return st;
        if (!last) std::swap(cur, nxt);
    }
    return MA_OK;
}

int run_muon_jobs(const MuonJob* jobs, int njobs, cudaStream_t s, int sms, int* launches) {
    if (njobs > ns_tc_max_jobs()) return MA_ERR_UNSUPPORTED;
    const int st = prep_jobs(jobs, njobs, s, 0, launches);
    return st ? st : chain_jobs(jobs, njobs, s, sms, launches);
}

// One batch with workspace ws.
int run_muon(int batch, const MuonGeom& g, float* const* W, const void* const* G, int gdt, float* const* M,
             const ma_muon_hparams_t& hp, void* ws, cudaStream_t s, int sms, int* launches) {
    const MuonJob j{batch, g, W, G, gdt, M, &hp, reinterpret_cast<uint8_t*>(ws)};
    return run_muon_jobs(&j, 1, s, sms, launches);
}

int check_ptr_array(const void* const* a, int n, size_t align) {
    if (!a) return MA_ERR_NULL;
    for (int i = 0; i < n; ++i) {
        if (!a[i]) return MA_ERR_NULL;
        if (!aligned(a[i], align)) return MA_ERR_ALIGN;
    }
    return MA_OK;
}

// MA_ERR_ARG if any two of the [begin, end) byte ranges overlap (buffers that
// one call writes must be disjoint). Sorts w.
int check_disjoint(std::vector<std::pair<uintptr_t, uintptr_t>>& w) {
    std::sort(w.begin(), w.end());
    for (size_t k = 1; k < w.size(); ++k)
        if (w[k].first < w[k - 1].second) return MA_ERR_ARG;
    return MA_OK;
}

int check_muon_call(int batch, int64_t R, int64_t C, float* const* W, const void* const* G, int gdt,
                    float* const* M, const ma_muon_hparams_t* hp, MuonGeom* g) {
    int st = check_muon_hp(hp);
    if (st) return st;
    if (batch < 0 || R < 0 || C < 0) return MA_ERR_SHAPE;
    if (batch > MA_MAX_BATCH) return MA_ERR_UNSUPPORTED;
    if (gdt != MA_F32 && gdt != MA_BF16) return MA_ERR_DTYPE;
    if ((st = muon_geom(batch, R, C, *hp, g))) return st;
    if (batch == 0 || R == 0 || C == 0) return MA_OK;
    if ((st = check_ptr_array(reinterpret_cast<const void* const*>(W), batch, 16))) return st;
    if ((st = check_ptr_array(G, batch, 16))) return st;
    if ((st = check_ptr_array(reinterpret_cast<const void* const*>(M), batch, 16))) return st;
    if (C % 8 != 0) return MA_ERR_ALIGN;
    if (g->units > 65535 || g->m > INT_MAX || g->n > INT_MAX || g->parts > INT_MAX) return MA_ERR_UNSUPPORTED;
    std::vector<std::pair<uintptr_t, uintptr_t>> w;
    const uintptr_t bytes = (uintptr_t)(R * C) * 4;
    for (int b = 0; b < batch; ++b) {
        w.push_back({(uintptr_t)W[b], (uintptr_t)W[b] + bytes});
        w.push_back({(uintptr_t)M[b], (uintptr_t)M[b] + bytes});
    }
    return check_disjoint(w);
}

// ------------------------------------------------------------------ AdamW helpers

AdamwGroupConst adamw_const(const ma_adamw_hparams_t& h) {
    AdamwGroupConst c;
    const double bc1 = 1.0 - std::pow((double)h.beta1, (double)h.step);
    const double bc2 = 1.0 - std::pow((double)h.beta2, (double)h.step);
    c.decay = (float)(1.0 - (double)h.lr * (double)h.weight_decay);
    c.step_size = (float)((double)h.lr / bc1);
    c.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
    c.beta1 = h.beta1;
    c.beta2 = h.beta2;
    c.omb1 = (float)(1.0 - (double)h.beta1);
    c.omb2 = (float)(1.0 - (double)h.beta2);
    c.eps = h.eps;
    return c;
}

int check_adamw_hp(const ma_adamw_hparams_t* h) {
    if (!h) return MA_ERR_NULL;
    if (h->step < 1) return MA_ERR_ARG;
    if (!(h->beta1 >= 0.f && h->beta1 < 1.f) || !(h->beta2 >= 0.f && h->beta2 < 1.f)) return MA_ERR_ARG;
    if (!(h->eps >= 0.f) || !std::isfinite(h->lr) || !std::isfinite(h->weight_decay)) return MA_ERR_ARG;
    return MA_OK;
}

struct AdamwItem {
    float* p;
    const void* g;
    float* m;
    float* v;
    int64_t numel;
    int group;
};

// Launch AdamW over items (all with gradient dtype gdt) in parameter-block batches.
int run_adamw(const std::vector<AdamwItem>& items, int gdt, const AdamwGroupConst* grp, int ngroups, cudaStream_t s,
              int* launches) {
    static thread_local AdamwLaunch L;  // ~19 KB parameter block, copied at launch
    size_t i = 0;
    while (i < items.size()) {
        std::memset(&L, 0, sizeof(L));
        L.gdt = gdt;
        L.status = device_status_ptr();
        for (int k = 0; k < ngroups; ++k) L.grp[k] = grp[k];
        int64_t chunk = 0;
        int nt = 0;
        while (i < items.size() && nt < kAdamwMaxTensorsPerLaunch) {
            const AdamwItem& it = items[i++];
            if (it.numel == 0) continue;
            AdamwTensorDesc& d = L.t[nt++];
            d.p = it.p;
            d.g = it.g;
            d.m = it.m;
            d.v = it.v;
            d.numel = it.numel;
            d.chunk0 = chunk;
            d.group = it.group;
            const size_t gal = gdt == MA_BF16 ? 8 : 16;
            d.vec = aligned(it.p, 16) && aligned(it.m, 16) && aligned(it.v, 16) && aligned(it.g, gal);
            chunk += (it.numel + kAdamwChunk - 1) / kAdamwChunk;
            if (chunk > (int64_t)INT_MAX - kAdamwMaxTensorsPerLaunch) break;
        }
        L.ntensors = nt;
        L.nchunks = chunk;
        if (nt > 0) {
            double elems = 0.0;
            for (int k = 0; k < nt; ++k) elems += (double)L.t[k].numel;
            const int pr = prof_begin(MA_PROF_ADAMW, s);
            cudaError_t e = launch_adamw(L, s);
            prof_end(pr, s, 0.0, elems * (gdt == MA_BF16 ? 26.0 : 28.0));
            if (e != cudaSuccess) return MA_ERR_CUDA;
            ++*launches;
        }
    }
    return MA_OK;
}

__global__ void wait_selftest_kernel(long long limit_ns, int* status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // nothing ever arrives on `bar`: this wait must give up after limit_ns
        mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns, status);
    }
    __syncthreads();
}

}  // namespace

cudaError_t launch_wait_selftest(long long limit_ns, int* status, cudaStream_t s) {
    wait_selftest_kernel<<<1, 32, 0, s>>>(limit_ns, status);
    return cudaGetLastError();
}

}  // namespace ma

// ====================================================================== C ABI

using namespace ma;

struct ma_plan {
    std::vector<ma_tensor_t> t;
    std::vector<int32_t> kind;
    std::vector<int32_t> group_kind;
    std::vector<int> adamw_idx;
    struct Bucket {
        int group;
        int64_t R, C;
        std::vector<int> members;
        int sub;  // matrices per sub-batch
    };
    std::vector<Bucket> buckets;
    size_t ws_bytes = 0;
    // > 0: the workspace holds two halves of this many bytes, used by the Muon
    // segments in turn, so that a segment's momentum pass can run under the
    // chain of the one before it (on the side stream)
    size_t region = 0;
    int last_launches = 0;
    std::vector<cudaEvent_t> events;  // segment-ready events of muonadamw_step_from_host
    cudaStream_t side = nullptr;      // the momentum passes that run under a chain
    int side_dev = -1;
    std::vector<cudaEvent_t> side_events;
    // muonadamw_step_graph: the captured step and the kernel nodes whose
    // parameters follow the per-step hyperparameters
    struct GraphNode {
        cudaGraphNode_t node;
        cudaKernelNodeParams params;  // func, launch shape; kernelParams replaced on update
        std::vector<uint8_t> arg;     // the kernel's single by-value parameter
        int final_apply;              // 0: AdamW launch, 1: Newton-Schulz final apply
    };
    struct Graph {
        cudaGraph_t graph = nullptr;
        cudaGraphExec_t exec = nullptr;
        cudaStream_t capture = nullptr;
        int capture_dev = -1;  // device of `capture`
        std::vector<uint8_t> key;
        std::vector<GraphNode> nodes;
        int launches = 0;
        int captures = 0;
        void release() {
            if (exec) cudaGraphExecDestroy(exec);
            if (graph) cudaGraphDestroy(graph);
            exec = nullptr;
            graph = nullptr;
            nodes.clear();
            key.clear();
        }
    } g;
    ~ma_plan() {
        for (cudaEvent_t e : events) cudaEventDestroy(e);
        for (cudaEvent_t e : side_events) cudaEventDestroy(e);
        g.release();
        if (g.capture) cudaStreamDestroy(g.capture);
        if (side) cudaStreamDestroy(side);
    }
};

namespace ma {
namespace {

// A unit of launch work inside one step: every AdamW tensor, or one or more
// Muon sub-batches (parts) whose Newton-Schulz steps share launches.
struct Part {
    int bucket, start, count;
};
struct Segment {
    int adamw;  // 1: the AdamW tensors; 0: Muon parts
    std::vector<Part> parts;
};

int64_t tensor_numel(const ma_tensor_t& x) {
    int64_t n = 1;
    for (int d = 0; d < x.ndim; ++d) n *= x.shape[d];
    return n;
}

// The workspace one Muon segment may use: half of the plan's workspace when
// it is split in two (see run_segments), else all of it.
size_t seg_limit(const ma_plan* plan) { return plan->region ? plan->region : plan->ws_bytes; }

// Shared checks of a step over a plan; fills *sms.
int check_step(ma_plan* plan, const ma_group_t* groups, void* ws, size_t ws_bytes, int* sms) {
    if (!plan) return MA_ERR_NULL;
    const int ngroups = (int)plan->group_kind.size();
    if (ngroups > 0 && !groups) return MA_ERR_NULL;
    int st;
    for (int k = 0; k < ngroups; ++k) {
        if (groups[k].kind != plan->group_kind[k]) return MA_ERR_ARG;
        if (groups[k].kind == MA_MUON) {
            if ((st = check_muon_hp(&groups[k].muon))) return st;
        } else if ((st = check_adamw_hp(&groups[k].adamw))) {
            return st;
        }
    }
    // the plan's bucket geometry depends on heads, steps, precision and c != 0
    for (auto& b : plan->buckets) {
        MuonGeom g;
        if ((st = muon_geom(b.sub, b.R, b.C, groups[b.group].muon, &g))) return st;
        if (g.total > seg_limit(plan)) return MA_ERR_ARG;
    }
    if (plan->ws_bytes > 0 && (!ws || !aligned(ws, kAlign) || ws_bytes < plan->ws_bytes)) return MA_ERR_WORKSPACE;
    *sms = 0;
    if (!plan->adamw_idx.empty() || !plan->buckets.empty()) {
        if ((st = device_ok_and_sms(sms))) return st;
    }
    return MA_OK;
}

size_t part_ws(const ma_plan* plan, const ma_group_t* groups, const Part& pt) {
    const auto& b = plan->buckets[pt.bucket];
    MuonGeom g;
    if (muon_geom(pt.count, b.R, b.C, groups[b.group].muon, &g)) return SIZE_MAX;
    return g.total;
}

// Segments in launch order. cap bounds the Muon sub-batch sizes (0 = the
// plan's own sub-batch size); with first_cap > 0 the first sub-batch holds at
// most first_cap matrices and each later one at most twice the one before,
// up to cap, so that the first copy of a host-gradient step is short. AdamW
// goes first or last. With
// group_limit > 0, consecutive sub-batches whose Newton-Schulz chains take
// the same kernels are merged into one segment while their summed workspace
// stays within group_limit and the launch tables have room (jobs, weights).
std::vector<Segment> step_segments(const ma_plan* plan, const ma_group_t* groups, int first_cap, int cap,
                                   bool adamw_last, size_t group_limit) {
    std::vector<Segment> segs;
    if (!adamw_last && !plan->adamw_idx.empty()) segs.push_back({1, {}});
    int ramp = first_cap;  // 0 once the ramp has reached cap
    size_t seg_ws = 0;
    int seg_w = 0;
    for (int bi = 0; bi < (int)plan->buckets.size(); ++bi) {
        const auto& b = plan->buckets[bi];
        const int nb = (int)b.members.size();
        for (int s0 = 0; s0 < nb;) {
            int lim = b.sub;
            if (cap > 0) lim = std::min(lim, cap);
            if (ramp > 0) lim = std::min(lim, ramp);
            const int cnt = std::min(lim, nb - s0);
            const Part pt{bi, s0, cnt};
            const size_t ws = part_ws(plan, groups, pt);
            const int nw = cnt;
            bool merge = false;
            if (group_limit > 0 && !segs.empty() && !segs.back().adamw) {
                const Segment& last = segs.back();
                const auto& lb = plan->buckets[last.parts.back().bucket];
                merge = ns_compatible(groups[lb.group].muon, groups[b.group].muon) &&
                        (int)last.parts.size() < ns_tc_max_jobs() && seg_w + nw <= ns_tc_max_weights() &&
                        ws <= group_limit && seg_ws <= group_limit - ws;
            }
            if (merge) {
                segs.back().parts.push_back(pt);
                seg_ws += ws;
                seg_w += nw;
            } else {
                segs.push_back({0, {pt}});
                seg_ws = ws;
                seg_w = nw;
            }
            s0 += cnt;
            if (ramp > 0) ramp = (cap > 0 && 2 * ramp >= cap) || ramp >= (1 << 20) ? 0 : 2 * ramp;
        }
    }
    if (adamw_last && !plan->adamw_idx.empty()) segs.push_back({1, {}});
    return segs;
}

// An NVTX range over a scope (host-side markers for timeline tools such as
// Nsight Systems; without a tool attached the calls do nothing).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

// The jobs of one Muon segment, with the pointer tables they point into.
struct SegJobs {
    std::vector<MuonJob> jobs;
    std::vector<float*> W, M;
    std::vector<const void*> G;
};

// Jobs of Muon segment sg with their workspaces laid out from base.
void build_jobs(const ma_plan* plan, const ma_group_t* groups, const Segment& sg, uint8_t* base, SegJobs& out) {
    const int np = (int)sg.parts.size();
    out.jobs.assign(np, MuonJob{});
    int total = 0;
    for (const Part& pt : sg.parts) total += pt.count;
    out.W.clear();
    out.M.clear();
    out.G.clear();
    out.W.reserve(total);  // no reallocation below: the jobs keep pointers into these tables
    out.M.reserve(total);
    out.G.reserve(total);
    for (int q = 0; q < np; ++q) {
        const Part& pt = sg.parts[q];
        const auto& b = plan->buckets[pt.bucket];
        const ma_muon_hparams_t& hp = groups[b.group].muon;
        MuonJob& J = out.jobs[q];
        J.batch = pt.count;
        muon_geom(pt.count, b.R, b.C, hp, &J.g);
        J.gdt = plan->t[b.members[0]].grad_dtype;
        J.hp = &hp;
        J.ws = base;
        base += J.g.total;  // a multiple of the workspace alignment
        const size_t off = out.W.size();
        for (int k = 0; k < pt.count; ++k) {
            const ma_tensor_t& x = plan->t[b.members[pt.start + k]];
            out.W.push_back(x.param);
            out.G.push_back(x.grad);
            out.M.push_back(x.state0);
        }
        J.W = out.W.data() + off;
        J.G = out.G.data() + off;
        J.M = out.M.data() + off;
    }
}

int run_adamw_segment(ma_plan* plan, const ma_group_t* groups, cudaStream_t s, int* launches) {
    NvtxRange range("ma.adamw");
    const int ngroups = (int)plan->group_kind.size();
    AdamwGroupConst gc[MA_MAX_GROUPS];
    std::memset(gc, 0, sizeof(gc));
    for (int k = 0; k < ngroups; ++k)
        if (groups[k].kind == MA_ADAMW) gc[k] = adamw_const(groups[k].adamw);
    int st;
    for (int dt = 0; dt < 2; ++dt) {
        std::vector<AdamwItem> items;
        for (int i : plan->adamw_idx) {
            const ma_tensor_t& x = plan->t[i];
            if (x.grad_dtype != dt) continue;
            items.push_back({x.param, x.grad, x.state0, x.state1, tensor_numel(x), x.group});
        }
        if (!items.empty() && (st = run_adamw(items, dt, gc, ngroups, s, launches))) return st;
    }
    return MA_OK;
}

// Whether a segment's momentum passes may run on the side stream under the
// Newton-Schulz chain of the segment before it: bf16 operands (both momentum
// kernels then fit beside a Newton-Schulz CTA on an SM).
bool side_prep_ok(const SegJobs& sj) {
    for (const MuonJob& j : sj.jobs)
        if (j.g.total > 0 && j.hp->precision) return false;
    return true;
}

// Whether a segment's chain runs on the tensor cores (the CTAs the side
// stream's momentum kernel is sized to run beside).
bool tc_chain(const SegJobs& sj) {
    for (const MuonJob& j : sj.jobs)
        if (j.g.total > 0 && j.hp->precision) return false;
    return true;
}

// The plan's side stream and an event pool on the current device.
int side_resources(ma_plan* plan, int dev, size_t nevents, cudaStream_t* side) {
    if (plan->side && plan->side_dev != dev) {
        int cur = dev;
        cudaSetDevice(plan->side_dev);
        cudaStreamDestroy(plan->side);
        for (cudaEvent_t e : plan->side_events) cudaEventDestroy(e);
        cudaSetDevice(cur);
        plan->side = nullptr;
        plan->side_events.clear();
    }
    if (!plan->side) {
        int lo = 0, hi = 0;
        if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return MA_ERR_CUDA;
        // the least priority: the Newton-Schulz kernels of the caller's stream go first
        if (cudaStreamCreateWithPriority(&plan->side, cudaStreamNonBlocking, lo) != cudaSuccess) return MA_ERR_CUDA;
        plan->side_dev = dev;
    }
    while (plan->side_events.size() < nevents) {
        cudaEvent_t e;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return MA_ERR_CUDA;
        plan->side_events.push_back(e);
    }
    *side = plan->side;
    return MA_OK;
}

// One step over segments, on stream s. ready (may be null): per segment, an
// event its work must wait for (the host copies of its gradients).
//
// With the plan's double workspace (plan->region > 0, only for plans made
// with ma_set_momentum_overlap on), the Muon segments use its two halves in
// turn, and the momentum pass of segment q + 1 runs on the plan's side
// stream, on a small grid that fits beside the Newton-Schulz CTAs, while
// segment q's chain runs. It is off by default: on a B200 the side blocks
// slow the CTA pairs they share SMs with by more than the pass costs inline,
// and every launch ends with its slowest pair. The side stream starts after
// all work queued on s before the step; segment q + 1's momentum pass waits
// for the chain of segment q - 1, the last user of its workspace half;
// segment q + 1's chain waits for its momentum pass; s waits for the side
// stream at the end. Every kernel does the same arithmetic as on one stream,
// so the results are the same bits.
int run_segments(ma_plan* plan, const ma_group_t* groups, const std::vector<Segment>& segs, void* ws, cudaStream_t s,
                 int sms, int* launches, const cudaEvent_t* ready) {
    std::vector<int> mi;  // Muon segments, in order
    for (int k = 0; k < (int)segs.size(); ++k)
        if (!segs[k].adamw) mi.push_back(k);
    const int nm = (int)mi.size();
    uint8_t* base = reinterpret_cast<uint8_t*>(ws);
    const size_t region = plan->region;
    std::vector<SegJobs> sj(nm);
    for (int q = 0; q < nm; ++q) build_jobs(plan, groups, segs[mi[q]], base + (region ? (q & 1) * region : 0), sj[q]);
    std::vector<char> on_side(nm, 0);
    bool any_side = false;
    for (int q = 1; q < nm && region; ++q) {
        on_side[q] = side_prep_ok(sj[q]) && tc_chain(sj[q - 1]);
        any_side = any_side || on_side[q];
    }
    cudaStream_t side = nullptr;
    cudaEvent_t *ev_fork = nullptr, *ev_prep = nullptr, *ev_chain = nullptr;
    int st;
    if (any_side) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return MA_ERR_CUDA;
        if ((st = side_resources(plan, dev, 2 + 2 * (size_t)nm, &side))) return st;
        ev_fork = &plan->side_events[0];
        ev_prep = &plan->side_events[1];
        ev_chain = &plan->side_events[1 + nm];
        if (cudaEventRecord(*ev_fork, s) != cudaSuccess || cudaStreamWaitEvent(side, *ev_fork, 0) != cudaSuccess)
            return MA_ERR_CUDA;
    }
    bool side_work = false;
    int q = 0;
    for (int k = 0; k < (int)segs.size(); ++k) {
        if (ready && cudaStreamWaitEvent(s, ready[k], 0) != cudaSuccess) return MA_ERR_CUDA;
        if (segs[k].adamw) {
            if ((st = run_adamw_segment(plan, groups, s, launches))) return st;
            continue;
        }
        NvtxRange range("ma.muon");
        SegJobs& cur = sj[q];
        if (!on_side[q]) {
            if ((st = prep_jobs(cur.jobs.data(), (int)cur.jobs.size(), s, 0, launches))) return st;
        } else if (cudaStreamWaitEvent(s, ev_prep[q], 0) != cudaSuccess) {
            return MA_ERR_CUDA;
        }
        if (q + 1 < nm && on_side[q + 1]) {
            SegJobs& nx = sj[q + 1];
            if (ready && cudaStreamWaitEvent(side, ready[mi[q + 1]], 0) != cudaSuccess) return MA_ERR_CUDA;
            if (q >= 1 && cudaStreamWaitEvent(side, ev_chain[q - 1], 0) != cudaSuccess) return MA_ERR_CUDA;
            // one block per SM: each sits beside that SM's Newton-Schulz CTA
            if ((st = prep_jobs(nx.jobs.data(), (int)nx.jobs.size(), side, sms, launches, true))) return st;
            if (cudaEventRecord(ev_prep[q + 1], side) != cudaSuccess) return MA_ERR_CUDA;
            side_work = true;
        }
        if ((st = chain_jobs(cur.jobs.data(), (int)cur.jobs.size(), s, sms, launches))) return st;
        if (any_side && cudaEventRecord(ev_chain[q], s) != cudaSuccess) return MA_ERR_CUDA;
        ++q;
    }
    if (side_work) {
        // join: s continues after everything queued on the side stream
        if (cudaEventRecord(*ev_fork, side) != cudaSuccess || cudaStreamWaitEvent(s, *ev_fork, 0) != cudaSuccess)
            return MA_ERR_CUDA;
    }
    return MA_OK;
}

}  // namespace
}  // namespace ma

extern "C" {

const char* ma_status_string(int s) {
    switch (s) {
        case MA_OK: return "ok";
        case MA_ERR_NULL: return "null pointer";
        case MA_ERR_SHAPE: return "bad shape or size";
        case MA_ERR_DTYPE: return "bad dtype";
        case MA_ERR_ALIGN: return "misaligned pointer or row length";
        case MA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case MA_ERR_UNSUPPORTED: return "unsupported request";
        case MA_ERR_CUDA: return "CUDA runtime error";
        case MA_ERR_TIMEOUT: return "device wait timed out";
        case MA_ERR_ARG: return "hyperparameter out of range";
        case MA_ERR_BOUNDS: return "guarded device index out of bounds (debug build)";
        default: return "unknown status";
    }
}

int ma_version(void) { return MA_VERSION; }

size_t ma_struct_size(int which) {
    switch (which) {
        case 0: return sizeof(ma_tensor_t);
        case 1: return sizeof(ma_group_t);
        case 2: return sizeof(ma_muon_hparams_t);
        case 3: return sizeof(ma_adamw_hparams_t);
        case 4: return sizeof(ma_shard_slot_t);
        case 5: return sizeof(ma_shard_bucket_t);
        default: return 0;
    }
}

int ma_partition(const ma_tensor_t* t, int n, int32_t* kind_out) {
    if (n < 0) return MA_ERR_SHAPE;
    if (n == 0) return MA_OK;
    if (!t || !kind_out) return MA_ERR_NULL;
    for (int i = 0; i < n; ++i) {
        if (t[i].ndim < 0) return MA_ERR_SHAPE;
        if (t[i].ndim >= 3) return MA_ERR_UNSUPPORTED;
        if (t[i].role < MA_ROLE_HIDDEN || t[i].role > MA_ROLE_FORCE_ADAMW) return MA_ERR_ARG;
    }
    for (int i = 0; i < n; ++i) {
        int k = MA_ADAMW;
        if (t[i].ndim == 2 && t[i].role == MA_ROLE_HIDDEN) k = MA_MUON;
        kind_out[i] = k;
    }
    return MA_OK;
}

int ma_assign_owners(const ma_tensor_t* t, int n, const ma_group_t* groups, int ngroups, int world_size,
                     int32_t* owner_out) {
    if (n < 0 || ngroups < 0) return MA_ERR_SHAPE;
    if (world_size < 1) return MA_ERR_ARG;
    if (n == 0) return MA_OK;
    if (!t || !owner_out || !groups) return MA_ERR_NULL;
    std::vector<int32_t> kind(n);
    int st = ma_partition(t, n, kind.data());
    if (st) return st;
    std::vector<double> cost(n, 0.0);
    for (int i = 0; i < n; ++i) {
        if (t[i].group < 0 || t[i].group >= ngroups) return MA_ERR_ARG;
        double numel = 1.0;
        for (int d = 0; d < t[i].ndim; ++d) {
            if (t[i].shape[d] < 0) return MA_ERR_SHAPE;
            numel *= (double)t[i].shape[d];
        }
        if (kind[i] == MA_MUON) {
            const ma_muon_hparams_t& hp = groups[t[i].group].muon;
            const int heads = hp.heads < 1 ? 1 : hp.heads;
            const double Rh = (double)t[i].shape[0] / heads, C = (double)t[i].shape[1];
            const double m = std::min(Rh, C), nn = std::max(Rh, C);
            const int steps = hp.ns_steps < 1 ? 1 : hp.ns_steps;
            cost[i] = heads * steps * (m * (m + 1) * nn + 2 * m * m * nn) + numel;
        } else {
            cost[i] = numel;
        }
    }
    for (int pass = 0; pass < 2; ++pass) {
        const int want = pass == 0 ? MA_MUON : MA_ADAMW;
        std::vector<int> idx;
        for (int i = 0; i < n; ++i)
            if (kind[i] == want) idx.push_back(i);
        std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return cost[a] > cost[b]; });
        std::vector<double> load(world_size, 0.0);
        for (int i : idx) {
            int best = 0;
            for (int r = 1; r < world_size; ++r)
                if (load[r] < load[best]) best = r;
            owner_out[i] = best;
            load[best] += cost[i];
        }
    }
    return MA_OK;
}

namespace {

int64_t shard_align(int64_t x) { return (x + MA_SHARD_ALIGN - 1) / MA_SHARD_ALIGN * MA_SHARD_ALIGN; }

struct ShardBucket {
    int first;                 // lowest tensor index in the bucket (orders the buckets)
    int kind;
    std::vector<int> members;  // tensor indices, ascending
};

}  // namespace

int ma_shard_layout(const ma_tensor_t* t, int n, const ma_group_t* groups, int ngroups, int world_size,
                    int64_t seg_cap, ma_shard_slot_t* slots, ma_shard_bucket_t* buckets, int* nbuckets,
                    int64_t* total) {
    if (n < 0 || ngroups < 0) return MA_ERR_SHAPE;
    if (world_size < 1 || seg_cap < 1) return MA_ERR_ARG;
    if (!nbuckets || !total) return MA_ERR_NULL;
    *nbuckets = 0;
    *total = 0;
    if (n == 0) return MA_OK;
    if (!t || !slots || !buckets || !groups) return MA_ERR_NULL;
    std::vector<int32_t> kind(n);
    int st = ma_partition(t, n, kind.data());
    if (st) return st;
    const int64_t kMaxElems = int64_t(1) << 50;
    std::vector<int64_t> numel(n, 1);
    for (int i = 0; i < n; ++i) {
        if (t[i].group < 0 || t[i].group >= ngroups) return MA_ERR_ARG;
        if (groups[t[i].group].kind != kind[i]) return MA_ERR_ARG;
        for (int d = 0; d < t[i].ndim; ++d) {
            if (t[i].shape[d] < 0 || t[i].shape[d] > kMaxElems) return MA_ERR_SHAPE;
            numel[i] *= t[i].shape[d];
            if (numel[i] > kMaxElems) return MA_ERR_SHAPE;
        }
    }

    // Muon, first pass: matrices of one shape and group, in order of
    // appearance, are cut into buckets of world_size * k matrices, k = as many
    // as fit one rank's segment cap (at least one). Matrix j of such a bucket
    // belongs to rank j % world_size, so every segment holds k matrices. The
    // last c % world_size matrices of a class of c are left over.
    std::vector<ShardBucket> bl;
    std::vector<int> leftover;
    std::vector<bool> placed(n, false);
    for (int i = 0; i < n; ++i) {
        if (kind[i] != MA_MUON || placed[i]) continue;
        std::vector<int> cls;
        for (int j = i; j < n; ++j)
            if (kind[j] == MA_MUON && !placed[j] && t[j].shape[0] == t[i].shape[0] &&
                t[j].shape[1] == t[i].shape[1] && t[j].group == t[i].group) {
                cls.push_back(j);
                placed[j] = true;
            }
        const size_t full = cls.size() / (size_t)world_size * (size_t)world_size;
        const int64_t a = shard_align(numel[i]);
        const int64_t per_rank = std::min<int64_t>(n, std::max<int64_t>(1, a > 0 ? seg_cap / a : seg_cap));
        const size_t k = (size_t)per_rank * (size_t)world_size;
        for (size_t b = 0; b < full; b += k) {
            ShardBucket sb{cls[b], MA_MUON, {}};
            for (size_t j = b; j < std::min(full, b + k); ++j) sb.members.push_back(cls[j]);
            bl.push_back(std::move(sb));
        }
        for (size_t j = full; j < cls.size(); ++j) leftover.push_back(cls[j]);
    }
    // Muon, second pass: the leftovers, in order of appearance, fill mixed
    // buckets; one closes before the matrix that would take the bucket's
    // average per-rank share past the cap. Their owners are set below,
    // largest matrix first onto the least-loaded rank.
    std::sort(leftover.begin(), leftover.end());
    {
        ShardBucket cur{-1, MA_MUON, {}};
        int64_t run = 0;
        for (int i : leftover) {
            const int64_t next = run + shard_align(numel[i]);
            if (!cur.members.empty() && (next + world_size - 1) / world_size > seg_cap) {
                bl.push_back(std::move(cur));
                cur = ShardBucket{-1, MA_MUON, {}};
                run = 0;
            }
            if (cur.members.empty()) cur.first = i;
            cur.members.push_back(i);
            run += shard_align(numel[i]);
            if (run > kMaxElems) return MA_ERR_SHAPE;
        }
        if (!cur.members.empty()) bl.push_back(std::move(cur));
    }
    // AdamW: tensors in order of appearance; a bucket closes before the
    // tensor that would take its per-rank share past the cap (a bucket always
    // takes at least one tensor). Its elements are split evenly by range.
    {
        ShardBucket cur{-1, MA_ADAMW, {}};
        int64_t run = 0;
        for (int i = 0; i < n; ++i) {
            if (kind[i] != MA_ADAMW) continue;
            const int64_t next = run + shard_align(numel[i]);
            if (!cur.members.empty() && (next + world_size - 1) / world_size > seg_cap) {
                bl.push_back(std::move(cur));
                cur = ShardBucket{-1, MA_ADAMW, {}};
                run = 0;
            }
            if (cur.members.empty()) cur.first = i;
            cur.members.push_back(i);
            run += shard_align(numel[i]);
            if (run > kMaxElems) return MA_ERR_SHAPE;
        }
        if (!cur.members.empty()) bl.push_back(std::move(cur));
    }
    std::stable_sort(bl.begin(), bl.end(), [](const ShardBucket& x, const ShardBucket& y) { return x.first < y.first; });

    // Owners and segment lengths first, so that an oversized layout is
    // refused before any output is written. A bucket whose matrices all share
    // one shape and whose count is a multiple of world_size is dealt round
    // robin; any other Muon bucket is packed largest first onto the
    // least-loaded rank (ties: lower rank, then lower tensor index). Within a
    // segment, matrices sit in order of appearance.
    std::vector<int> owner(n, -1);
    std::vector<int64_t> segs(bl.size());
    int64_t end = 0;
    for (size_t b = 0; b < bl.size(); ++b) {
        const ShardBucket& sb = bl[b];
        if (sb.kind == MA_MUON) {
            bool uniform = sb.members.size() % (size_t)world_size == 0;
            for (int i : sb.members)
                uniform = uniform && t[i].shape[0] == t[sb.members[0]].shape[0] &&
                          t[i].shape[1] == t[sb.members[0]].shape[1];
            std::vector<int64_t> load(world_size, 0);
            if (uniform) {
                for (size_t j = 0; j < sb.members.size(); ++j) {
                    owner[sb.members[j]] = (int)(j % (size_t)world_size);
                    load[j % (size_t)world_size] += shard_align(numel[sb.members[j]]);
                }
            } else {
                std::vector<int> order = sb.members;
                std::stable_sort(order.begin(), order.end(),
                                 [&](int x, int y) { return numel[x] > numel[y]; });
                for (int i : order) {
                    int r = 0;
                    for (int q = 1; q < world_size; ++q)
                        if (load[q] < load[r]) r = q;
                    owner[i] = r;
                    load[r] += shard_align(numel[i]);
                }
            }
            segs[b] = *std::max_element(load.begin(), load.end());
        } else {
            int64_t len = 0;
            for (int i : sb.members) len += shard_align(numel[i]);
            segs[b] = shard_align((len + world_size - 1) / world_size);
        }
        if (segs[b] > kMaxElems / world_size) return MA_ERR_SHAPE;
        end += segs[b] * world_size;
        if (end > kMaxElems) return MA_ERR_SHAPE;
    }
    int64_t start = 0;
    for (size_t b = 0; b < bl.size(); ++b) {
        const ShardBucket& sb = bl[b];
        const int64_t seg = segs[b];
        if (sb.kind == MA_MUON) {
            std::vector<int64_t> fill(world_size, 0);
            for (int i : sb.members) {
                const int r = owner[i];
                slots[i] = ma_shard_slot_t{(int32_t)b, r, start + r * seg + fill[r]};
                fill[r] += shard_align(numel[i]);
            }
        } else {
            int64_t off = 0;
            for (int i : sb.members) {
                slots[i] = ma_shard_slot_t{(int32_t)b, -1, start + off};
                off += shard_align(numel[i]);
            }
        }
        buckets[b] = ma_shard_bucket_t{sb.kind, (int32_t)sb.members.size(), start, seg};
        start += seg * world_size;
    }
    *nbuckets = (int)bl.size();
    *total = start;
    return MA_OK;
}

size_t muon_workspace_bytes(int batch, int64_t R, int64_t C, const ma_muon_hparams_t* hp) {
    if (check_muon_hp(hp) != MA_OK) return SIZE_MAX;
    MuonGeom g;
    if (muon_geom(batch, R, C, *hp, &g) != MA_OK) return SIZE_MAX;
    return g.total;
}

int muon_step_batched(int batch, int64_t R, int64_t C, float* const* W, const void* const* G, int gdt,
                      float* const* M, const ma_muon_hparams_t* hp, void* ws, size_t ws_bytes, void* stream) {
    MuonGeom g;
    int st = check_muon_call(batch, R, C, W, G, gdt, M, hp, &g);
    if (st) return st;
    if (g.total == 0) return MA_OK;
    if (!ws || !aligned(ws, kAlign) || ws_bytes < g.total) return MA_ERR_WORKSPACE;
    int sms = 0;
    if ((st = device_ok_and_sms(&sms))) return st;
    // a large batch runs as consecutive sub-batches of at most kSubBatchBytes of
    // workspace each (fewer units per launch; the workspace is reused)
    int sub = batch;
    MuonGeom gs = g;
    while (gs.total > kSubBatchBytes && sub > 1) {
        sub = std::max(1, sub / 2);
        muon_geom(sub, R, C, *hp, &gs);
    }
    int launches = 0;
    for (int s0 = 0; s0 < batch; s0 += sub) {
        const int cnt = std::min(sub, batch - s0);
        MuonGeom gc;
        muon_geom(cnt, R, C, *hp, &gc);
        if ((st = run_muon(cnt, gc, W + s0, G + s0, gdt, M + s0, *hp, ws, reinterpret_cast<cudaStream_t>(stream),
                           sms, &launches)))
            return st;
    }
    return MA_OK;
}

size_t ns_iterate_workspace_bytes(int batch, int64_t m, int64_t n) {
    if (batch < 0 || m < 0 || n < 0) return SIZE_MAX;
    const size_t x = align_up((size_t)batch * m * n * 2, kAlign);
    const size_t gm = align_up((size_t)batch * m * round8(m) * 2, kAlign);
    return x + 2 * gm;
}

int ns_iterate_bf16(int batch, int64_t m, int64_t n, const uint16_t* X_in, uint16_t* X_out, const float* coeffs,
                    int n_coeffs, int steps, void* ws, size_t ws_bytes, void* stream) {
    if (batch < 0 || m < 0 || n < 0) return MA_ERR_SHAPE;
    if (steps < 1 || steps > MA_MAX_NS_STEPS || !(n_coeffs == 1 || n_coeffs == steps)) return MA_ERR_ARG;
    if (!coeffs) return MA_ERR_NULL;
    for (int k = 0; k < 3 * n_coeffs; ++k)
        if (!std::isfinite(coeffs[k])) return MA_ERR_ARG;
    if (batch == 0 || m == 0 || n == 0) return MA_OK;
    if (!X_in || !X_out) return MA_ERR_NULL;
    if (m > n) return MA_ERR_SHAPE;
    if (n % 8 != 0 || !aligned(X_in, 16) || !aligned(X_out, 16)) return MA_ERR_ALIGN;
    if (batch > 65535 || n > INT_MAX) return MA_ERR_UNSUPPORTED;
    const size_t need = ns_iterate_workspace_bytes(batch, m, n);
    if (!ws || !aligned(ws, kAlign) || ws_bytes < need) return MA_ERR_WORKSPACE;
    int sms = 0;
    int st = device_ok_and_sms(&sms);
    if (st) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* base = reinterpret_cast<uint8_t*>(ws);
    void* T = base;
    void* Gb = base + align_up((size_t)batch * m * n * 2, kAlign);
    void* G2 = reinterpret_cast<uint8_t*>(Gb) + align_up((size_t)batch * m * round8(m) * 2, kAlign);
    NsParams p;
    std::memset(&p, 0, sizeof(p));
    p.units = batch;
    p.m = (int)m;
    p.n = (int)n;
    p.ldx = n;
    p.ldg = round8(m);
    p.x_unit = m * n;
    p.g_unit = m * round8(m);
    p.first = 0;
    p.heads = 1;
    p.wait_limit_ns = host_wait_limit_ns();
    p.status = device_status_ptr();
    const void* cur = X_in;
    for (int k = 0; k < steps; ++k) {
        const float* cf = coeffs + 3 * (n_coeffs == 1 ? 0 : k);
        p.a = cf[0];
        p.b = cf[1];
        p.c = cf[2];
        const bool quint = cf[2] != 0.f;
        p.coef_gram = quint ? 1.f : cf[1];
        auto launch = [&](int mode, const void* xb, const void* gb) -> int {
            const int pr = prof_begin(ns_prof_class(mode), s);
            cudaError_t e = launch_ns_tc(mode, p, xb, gb, sms, s);
            prof_end(pr, s, ns_flops(mode, batch, m, n), 0.0);
            return cuda_status(e);
        };
        p.out = Gb;
        if (launch(NS_GRAM, cur, Gb)) return MA_ERR_CUDA;
        void* Bbuf = Gb;
        if (quint) {
            p.xin = Gb;
            p.out = G2;
            if (launch(NS_GRAMSQ, cur, Gb)) return MA_ERR_CUDA;
            Bbuf = G2;
        }
        // the last iteration writes X_out; earlier ones alternate so that no GEMM
        // reads and writes the same buffer
        void* dst = ((steps - 1 - k) % 2 == 0) ? static_cast<void*>(X_out) : T;
        p.xin = cur;
        p.out = dst;
        if (launch(NS_APPLY, cur, Bbuf)) return MA_ERR_CUDA;
        cur = dst;
    }
    return MA_OK;
}

int adamw_step_fused(int n, float* const* P, const void* const* G, int gdt, float* const* M, float* const* V,
                     const int64_t* numel, const ma_adamw_hparams_t* hp, void* stream) {
    if (n < 0) return MA_ERR_SHAPE;
    int st = check_adamw_hp(hp);
    if (st) return st;
    if (gdt != MA_F32 && gdt != MA_BF16) return MA_ERR_DTYPE;
    if (n == 0) return MA_OK;
    if (!P || !G || !M || !V || !numel) return MA_ERR_NULL;
    std::vector<AdamwItem> items;
    items.reserve(n);
    for (int i = 0; i < n; ++i) {
        if (numel[i] < 0) return MA_ERR_SHAPE;
        if (numel[i] == 0) continue;
        if (!P[i] || !G[i] || !M[i] || !V[i]) return MA_ERR_NULL;
        if (!aligned(P[i], 4) || !aligned(M[i], 4) || !aligned(V[i], 4) || !aligned(G[i], gdt == MA_BF16 ? 2 : 4))
            return MA_ERR_ALIGN;
        items.push_back({P[i], G[i], M[i], V[i], numel[i], 0});
    }
    if (items.empty()) return MA_OK;
    std::vector<std::pair<uintptr_t, uintptr_t>> w;
    for (const AdamwItem& it : items) {
        const uintptr_t bytes = (uintptr_t)it.numel * 4;
        for (const float* q : {it.p, it.m, it.v}) w.push_back({(uintptr_t)q, (uintptr_t)q + bytes});
    }
    if ((st = check_disjoint(w))) return st;
    if ((st = device_ok_and_sms(nullptr))) return st;
    AdamwGroupConst c = adamw_const(*hp);
    int launches = 0;
    return run_adamw(items, gdt, &c, 1, reinterpret_cast<cudaStream_t>(stream), &launches);
}

int ma_plan_create(const ma_tensor_t* t, int n, const ma_group_t* groups, int ngroups, ma_plan_t** out,
                   size_t* ws_bytes) {
    if (!out || !ws_bytes) return MA_ERR_NULL;
    *out = nullptr;
    if (n < 0 || ngroups < 0) return MA_ERR_SHAPE;
    if (ngroups > MA_MAX_GROUPS) return MA_ERR_UNSUPPORTED;
    if ((n > 0 && !t) || (ngroups > 0 && !groups)) return MA_ERR_NULL;
    const size_t cap = *ws_bytes;
    std::vector<int32_t> kind(n);
    int st = ma_partition(t, n, kind.data());
    if (st) return st;
    for (int k = 0; k < ngroups; ++k) {
        if (groups[k].kind == MA_MUON) {
            if ((st = check_muon_hp(&groups[k].muon))) return st;
        } else if (groups[k].kind == MA_ADAMW) {
            if ((st = check_adamw_hp(&groups[k].adamw))) return st;
        } else {
            return MA_ERR_ARG;
        }
    }
    ma_plan* plan = new (std::nothrow) ma_plan();
    if (!plan) return MA_ERR_UNSUPPORTED;
    plan->t.assign(t, t + n);
    plan->kind = kind;
    for (int k = 0; k < ngroups; ++k) plan->group_kind.push_back(groups[k].kind);
    auto fail = [&](int code) {
        delete plan;
        return code;
    };
    for (int i = 0; i < n; ++i) {
        const ma_tensor_t& x = t[i];
        if (x.group < 0 || x.group >= ngroups) return fail(MA_ERR_ARG);
        if (groups[x.group].kind != kind[i]) return fail(MA_ERR_ARG);
        if (x.grad_dtype != MA_F32 && x.grad_dtype != MA_BF16) return fail(MA_ERR_DTYPE);
        int64_t numel = 1;
        for (int d = 0; d < x.ndim; ++d) {
            if (x.shape[d] < 0) return fail(MA_ERR_SHAPE);
            numel *= x.shape[d];
        }
        if (numel == 0) continue;
        if (!x.param || !x.grad || !x.state0) return fail(MA_ERR_NULL);
        if (kind[i] == MA_ADAMW) {
            if (!x.state1) return fail(MA_ERR_NULL);
            if (!aligned(x.param, 4) || !aligned(x.state0, 4) || !aligned(x.state1, 4) ||
                !aligned(x.grad, x.grad_dtype == MA_BF16 ? 2 : 4))
                return fail(MA_ERR_ALIGN);
            plan->adamw_idx.push_back(i);
        } else {
            if (!aligned(x.param, 16) || !aligned(x.state0, 16) || !aligned(x.grad, 16)) return fail(MA_ERR_ALIGN);
            if (x.shape[1] % 8 != 0) return fail(MA_ERR_ALIGN);
            const ma_muon_hparams_t& hp = groups[x.group].muon;
            if (x.shape[0] % hp.heads != 0) return fail(MA_ERR_SHAPE);
            bool found = false;
            for (auto& b : plan->buckets) {
                if (b.group == x.group && b.R == x.shape[0] && b.C == x.shape[1]) {
                    // one gradient dtype per bucket: a different dtype starts a new bucket
                    if (t[b.members[0]].grad_dtype != x.grad_dtype) continue;
                    b.members.push_back(i);
                    found = true;
                    break;
                }
            }
            if (!found) plan->buckets.push_back({x.group, x.shape[0], x.shape[1], {i}, 0});
        }
    }
    // Buffers the step writes (params and optimizer state) must not overlap:
    // a tensor listed twice, or state sharing memory with a parameter, would be
    // updated twice or read after being overwritten.
    {
        std::vector<std::pair<uintptr_t, uintptr_t>> w;  // [begin, end) of every written buffer
        for (int i = 0; i < n; ++i) {
            const int64_t numel = tensor_numel(t[i]);
            if (numel == 0) continue;
            const uintptr_t bytes = (uintptr_t)numel * 4;
            w.push_back({(uintptr_t)t[i].param, (uintptr_t)t[i].param + bytes});
            w.push_back({(uintptr_t)t[i].state0, (uintptr_t)t[i].state0 + bytes});
            if (kind[i] == MA_ADAMW) w.push_back({(uintptr_t)t[i].state1, (uintptr_t)t[i].state1 + bytes});
        }
        if ((st = check_disjoint(w))) return fail(st);
    }
    // Sub-batch sizes for a per-segment workspace budget `target` (halving a
    // bucket's sub-batch until it fits), then the workspace the step's
    // segments need (small buckets share Newton-Schulz launches within
    // `group` bytes) and how many Muon segments a step has. Returns nonzero
    // when a bucket does not fit even one matrix at a time.
    auto size_plan = [&](size_t target, size_t group, size_t* need_out, int* nseg) -> int {
        size_t need = 0;
        for (auto& b : plan->buckets) {
            const ma_muon_hparams_t& hp = groups[b.group].muon;
            const int nb = (int)b.members.size();
            int sub = std::min(nb, (int)MA_MAX_BATCH);
            MuonGeom g;
            int r = muon_geom(sub, b.R, b.C, hp, &g);
            if (r) return r;
            while (g.total > target && sub > 1) {
                sub = std::max(1, sub / 2);
                muon_geom(sub, b.R, b.C, hp, &g);
            }
            if (g.total > target) return MA_ERR_WORKSPACE;
            if (g.units > 65535 || g.m > INT_MAX || g.n > INT_MAX || g.parts > INT_MAX) return MA_ERR_UNSUPPORTED;
            b.sub = sub;
            need = std::max(need, g.total);
        }
        const size_t limit = group ? group : std::max(need, kGroupWsBytes);
        int muon_segments = 0;
        for (const Segment& sg : step_segments(plan, groups, 0, 0, false, limit)) {
            size_t tot = 0;
            for (const Part& pt : sg.parts) tot += part_ws(plan, groups, pt);
            need = std::max(need, tot);
            muon_segments += sg.adamw ? 0 : 1;
        }
        *need_out = need;
        *nseg = muon_segments;
        return MA_OK;
    };
    // With momentum overlap on, a step with two or more Muon segments gets a
    // workspace of two halves, so that one segment's momentum pass can run
    // under the chain of the one before it: without a cap, halves of at most
    // kSubBatchBytes (the sub-batch budget) each; with a cap, halves of at
    // most half the cap when every bucket fits in that, else one workspace of
    // at most the cap. Otherwise one workspace, sub-batches within
    // kSubBatchBytes or the cap.
    const bool halves = g_momentum_overlap.load(std::memory_order_relaxed) != 0;
    size_t need = 0;
    int nseg = 0;
    if (cap == 0) {
        if ((st = size_plan(kSubBatchBytes, 0, &need, &nseg))) return fail(st);
    } else if (!halves || size_plan(cap / 2, cap / 2, &need, &nseg) != MA_OK || nseg < 2) {
        if ((st = size_plan(cap, cap, &need, &nseg))) return fail(st);
        nseg = 0;  // no halves: one workspace within the cap
    }
    plan->ws_bytes = need;
    if (halves && nseg >= 2 && need > 0) {
        plan->region = align_up(need, kAlign);
        plan->ws_bytes = 2 * plan->region;
    }
    *ws_bytes = plan->ws_bytes;
    *out = plan;
    return MA_OK;
}

int muonadamw_step(ma_plan_t* plan, const ma_group_t* groups, void* ws, size_t ws_bytes, void* stream) {
    ma::NvtxRange range("ma.step");
    int sms = 0;
    int st = check_step(plan, groups, ws, ws_bytes, &sms);
    if (st) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int launches = 0;
    st = run_segments(plan, groups, step_segments(plan, groups, 0, 0, false, seg_limit(plan)), ws, s, sms, &launches,
                      nullptr);
    if (st) return st;
    plan->last_launches = launches;
    return MA_OK;
}

}  // extern "C"

namespace ma {
namespace {

// What a captured step depends on beyond the per-step values that are patched
// into its nodes (AdamW hyperparameters and step, Muon lr and weight decay on
// the tensor-core path): the workspace, the device and the rest of every Muon
// group's hyperparameters.
std::vector<uint8_t> graph_key(const ma_plan* plan, const ma_group_t* groups, const void* ws, int dev) {
    std::vector<uint8_t> k;
    auto put = [&k](const void* p, size_t n) {
        const uint8_t* b = reinterpret_cast<const uint8_t*>(p);
        k.insert(k.end(), b, b + n);
    };
    put(&ws, sizeof(ws));
    put(&dev, sizeof(dev));
    for (size_t i = 0; i < plan->group_kind.size(); ++i) {
        put(&groups[i].kind, sizeof(groups[i].kind));
        if (groups[i].kind != MA_MUON) continue;
        const ma_muon_hparams_t& h = groups[i].muon;
        const float lr = h.precision ? h.lr : 0.f, wd = h.precision ? h.weight_decay : 0.f;
        put(&lr, sizeof(lr));
        put(&wd, sizeof(wd));
        put(&h.beta, sizeof(h.beta));
        put(&h.eps, sizeof(h.eps));
        put(&h.nesterov, sizeof(h.nesterov));
        put(&h.ns_steps, sizeof(h.ns_steps));
        put(&h.n_coeffs, sizeof(h.n_coeffs));
        for (int c = 0; c < h.n_coeffs && c < MA_MAX_NS_STEPS; ++c) put(h.coeffs[c], 3 * sizeof(float));
        put(&h.scale_mode, sizeof(h.scale_mode));
        put(&h.heads, sizeof(h.heads));
        put(&h.precision, sizeof(h.precision));
        put(&h.cautious, sizeof(h.cautious));
    }
    return k;
}

struct FinalPatchCtx {
    const ma_plan* plan;
    const ma_group_t* groups;
    std::unordered_map<const float*, int> tensor_of;  // Muon weight -> table index
};

// The decay terms of one final-apply job, as run_muon_jobs computes them.
int patch_final_job(void* ctx, const float* W, int64_t Rh, int64_t C, float* decay, float* lr_s, float* lr_wd) {
    const FinalPatchCtx& c = *reinterpret_cast<const FinalPatchCtx*>(ctx);
    const auto it = c.tensor_of.find(W);
    if (it == c.tensor_of.end()) return MA_ERR_ARG;
    const ma_muon_hparams_t& hp = c.groups[c.plan->t[it->second].group].muon;
    *decay = 1.f - hp.lr * hp.weight_decay;
    *lr_s = hp.lr * shape_scale(Rh, C, hp.scale_mode);
    *lr_wd = hp.lr * hp.weight_decay;
    return MA_OK;
}

// Write this step's hyperparameters into the captured AdamW and final-apply nodes.
int graph_patch(ma_plan* plan, const ma_group_t* groups) {
    const int ngroups = (int)plan->group_kind.size();
    AdamwGroupConst gc[MA_MAX_GROUPS];
    std::memset(gc, 0, sizeof(gc));
    for (int k = 0; k < ngroups; ++k)
        if (groups[k].kind == MA_ADAMW) gc[k] = adamw_const(groups[k].adamw);
    FinalPatchCtx ctx{plan, groups, {}};
    for (size_t i = 0; i < plan->t.size(); ++i)
        if (plan->kind[i] == MA_MUON) ctx.tensor_of[plan->t[i].param] = (int)i;
    for (ma_plan::GraphNode& n : plan->g.nodes) {
        if (n.final_apply == 1) {
            const int st = ns_tc_patch_final(n.arg.data(), patch_final_job, &ctx);
            if (st) return st;
        } else {
            AdamwLaunch* L = reinterpret_cast<AdamwLaunch*>(n.arg.data());
            for (int k = 0; k < ngroups; ++k) L->grp[k] = gc[k];
        }
        cudaKernelNodeParams p = n.params;
        void* args[1] = {n.arg.data()};
        p.kernelParams = args;
        p.extra = nullptr;
        if (cudaGraphExecKernelNodeSetParams(plan->g.exec, n.node, &p) != cudaSuccess) return MA_ERR_CUDA;
    }
    return MA_OK;
}

// Capture one whole step on the plan's own stream and instantiate it.
int graph_capture(ma_plan* plan, const ma_group_t* groups, void* ws, int sms, int dev) {
    ma_plan::Graph& G = plan->g;
    G.release();
    if (G.capture && G.capture_dev != dev) {
        int cur = dev;
        cudaSetDevice(G.capture_dev);
        cudaStreamDestroy(G.capture);
        cudaSetDevice(cur);
        G.capture = nullptr;
    }
    if (!G.capture) {
        if (cudaStreamCreateWithFlags(&G.capture, cudaStreamNonBlocking) != cudaSuccess) return MA_ERR_CUDA;
        G.capture_dev = dev;
    }
    // everything that must not happen inside a capture: attribute set-up,
    // driver entry points, the status-word address, the side stream
    if (ns_tc_setup(sms) != cudaSuccess || prep_setup() != cudaSuccess || !device_status_ptr()) return MA_ERR_CUDA;
    if (plan->region) {
        size_t nm = 0;
        for (const Segment& sg : step_segments(plan, groups, 0, 0, false, seg_limit(plan))) nm += sg.adamw ? 0 : 1;
        cudaStream_t side;
        const int st0 = side_resources(plan, dev, 2 + 2 * nm, &side);
        if (st0) return st0;
    }
    const bool prof = g_prof_on;
    g_prof_on = false;
    if (cudaStreamBeginCapture(G.capture, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        g_prof_on = prof;
        return MA_ERR_CUDA;
    }
    int launches = 0;
    const int st =
        run_segments(plan, groups, step_segments(plan, groups, 0, 0, false, seg_limit(plan)), ws, G.capture, sms,
                     &launches, nullptr);
    cudaGraph_t graph = nullptr;
    const cudaError_t ec = cudaStreamEndCapture(G.capture, &graph);
    g_prof_on = prof;
    if (st || ec != cudaSuccess) {
        if (graph) cudaGraphDestroy(graph);
        return st ? st : MA_ERR_CUDA;
    }
    G.graph = graph;
    if (cudaGraphInstantiate(&G.exec, graph, 0) != cudaSuccess) {
        G.release();
        return MA_ERR_CUDA;
    }
    size_t n = 0;
    if (cudaGraphGetNodes(graph, nullptr, &n) != cudaSuccess) {
        G.release();
        return MA_ERR_CUDA;
    }
    std::vector<cudaGraphNode_t> nodes(n);
    if (n > 0 && cudaGraphGetNodes(graph, nodes.data(), &n) != cudaSuccess) {
        G.release();
        return MA_ERR_CUDA;
    }
    for (cudaGraphNode_t node : nodes) {
        cudaGraphNodeType type;
        if (cudaGraphNodeGetType(node, &type) != cudaSuccess || type != cudaGraphNodeTypeKernel) continue;
        cudaKernelNodeParams p;
        if (cudaGraphKernelNodeGetParams(node, &p) != cudaSuccess) {
            G.release();
            return MA_ERR_CUDA;
        }
        const bool adamw = p.func == adamw_kernel_func();
        const bool fin = ns_tc_is_final(p.func);
        if (!adamw && !fin) continue;
        const size_t bytes = adamw ? sizeof(AdamwLaunch) : ns_tc_launch_bytes();
        const uint8_t* a = reinterpret_cast<const uint8_t*>(p.kernelParams[0]);
        G.nodes.push_back({node, p, std::vector<uint8_t>(a, a + bytes), fin ? 1 : 0});
    }
    G.launches = launches;
    ++G.captures;
    return MA_OK;
}

}  // namespace
}  // namespace ma

extern "C" {

int muonadamw_step_graph(ma_plan_t* plan, const ma_group_t* groups, void* ws, size_t ws_bytes, void* stream) {
    int sms = 0;
    int st = check_step(plan, groups, ws, ws_bytes, &sms);
    if (st) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MA_ERR_CUDA;
    std::vector<uint8_t> key = graph_key(plan, groups, ws, dev);
    if (!plan->g.exec || key != plan->g.key) {
        if ((st = graph_capture(plan, groups, ws, sms, dev))) return st;
        plan->g.key = std::move(key);
    } else if ((st = graph_patch(plan, groups))) {
        return st;
    }
    if (cudaGraphLaunch(plan->g.exec, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MA_ERR_CUDA;
    plan->last_launches = plan->g.launches;
    return MA_OK;
}

int muonadamw_step_from_host(ma_plan_t* plan, const ma_group_t* groups, const void* const* host_grads, void* ws,
                             size_t ws_bytes, void* stream, void* copy_stream) {
    int sms = 0;
    int st = check_step(plan, groups, ws, ws_bytes, &sms);
    if (st) return st;
    const int n = (int)plan->t.size();
    if (n > 0 && !host_grads) return MA_ERR_NULL;
    for (int i = 0; i < n; ++i)
        if (tensor_numel(plan->t[i]) > 0 && !host_grads[i]) return MA_ERR_NULL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(copy_stream);
    // Muon sub-batches first (2, 4, 8, ... matrices, so the compute starts
    // early), the AdamW tensors last: every later copy overlaps earlier compute.
    const std::vector<Segment> segs = step_segments(plan, groups, kFromHostFirstBatch, kFromHostBatch, true, 0);
    while (plan->events.size() < segs.size() + 1) {
        cudaEvent_t e;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return MA_ERR_CUDA;
        plan->events.push_back(e);
    }
    // the copies overwrite the device gradients: wait for earlier work on `stream`
    cudaEvent_t prior = plan->events[segs.size()];
    if (cudaEventRecord(prior, s) != cudaSuccess || cudaStreamWaitEvent(cs, prior, 0) != cudaSuccess)
        return MA_ERR_CUDA;
    auto copy_tensor = [&](int i) -> int {
        const ma_tensor_t& x = plan->t[i];
        const size_t bytes = (size_t)tensor_numel(x) * (x.grad_dtype == MA_BF16 ? 2 : 4);
        if (bytes == 0) return MA_OK;
        return cudaMemcpyAsync(const_cast<void*>(x.grad), host_grads[i], bytes, cudaMemcpyHostToDevice, cs) ==
                       cudaSuccess
                   ? MA_OK
                   : MA_ERR_CUDA;
    };
    for (size_t k = 0; k < segs.size(); ++k) {
        const Segment& sg = segs[k];
        if (sg.adamw) {
            for (int i : plan->adamw_idx)
                if ((st = copy_tensor(i))) return st;
        } else {
            for (const Part& pt : sg.parts)
                for (int j = 0; j < pt.count; ++j)
                    if ((st = copy_tensor(plan->buckets[pt.bucket].members[pt.start + j]))) return st;
        }
        if (cudaEventRecord(plan->events[k], cs) != cudaSuccess) return MA_ERR_CUDA;
    }
    int launches = 0;
    if ((st = run_segments(plan, groups, segs, ws, s, sms, &launches, plan->events.data()))) return st;
    plan->last_launches = launches;
    return MA_OK;
}

int ma_plan_last_launches(const ma_plan_t* plan) { return plan ? plan->last_launches : 0; }

int ma_plan_graph_captures(const ma_plan_t* plan) { return plan ? plan->g.captures : 0; }

int ma_plan_describe(const ma_plan_t* plan, const ma_group_t* groups, char* buf, size_t len) {
    if (!plan || !buf || len == 0) return MA_ERR_NULL;
    const int ngroups = (int)plan->group_kind.size();
    if (ngroups > 0 && !groups) return MA_ERR_NULL;
    for (int k = 0; k < ngroups; ++k) {
        if (groups[k].kind != plan->group_kind[k]) return MA_ERR_ARG;
        if (groups[k].kind == MA_MUON && check_muon_hp(&groups[k].muon)) return MA_ERR_ARG;
    }
    std::string out;
    char line[256];
    int64_t adamw_elems = 0;
    for (int i : plan->adamw_idx) adamw_elems += tensor_numel(plan->t[i]);
    if (plan->region)
        std::snprintf(line, sizeof(line),
                      "workspace %zu bytes in two halves of %zu (momentum passes under the previous chain); "
                      "AdamW: %zu tensors, %lld elements\n",
                      plan->ws_bytes, plan->region, plan->adamw_idx.size(), (long long)adamw_elems);
    else
        std::snprintf(line, sizeof(line), "workspace %zu bytes; AdamW: %zu tensors, %lld elements\n", plan->ws_bytes,
                      plan->adamw_idx.size(), (long long)adamw_elems);
    out += line;
    for (size_t bi = 0; bi < plan->buckets.size(); ++bi) {
        const auto& b = plan->buckets[bi];
        const ma_muon_hparams_t& hp = groups[b.group].muon;
        MuonGeom g;
        muon_geom(b.sub, b.R, b.C, hp, &g);
        std::snprintf(line, sizeof(line), "bucket %zu: group %d, %lld x %lld, %zu matrices (%s grads), heads %d, "
                      "sub-batches of %d, %s\n", bi, b.group, (long long)b.R, (long long)b.C, b.members.size(),
                      plan->t[b.members[0]].grad_dtype == MA_BF16 ? "bf16" : "fp32", hp.heads, b.sub,
                      g.gspace ? "Gram-space chain" : "direct chain");
        out += line;
    }
    int si = 0;
    for (const Segment& sg : step_segments(plan, groups, 0, 0, false, seg_limit(plan))) {
        if (sg.adamw) {
            std::snprintf(line, sizeof(line), "segment %d: AdamW\n", si++);
            out += line;
            continue;
        }
        std::snprintf(line, sizeof(line), "segment %d: Newton-Schulz launches shared by", si++);
        out += line;
        for (const Part& pt : sg.parts) {
            std::snprintf(line, sizeof(line), " [bucket %d, matrices %d..%d]", pt.bucket, pt.start,
                          pt.start + pt.count - 1);
            out += line;
        }
        out += "\n";
    }
    const size_t n = std::min(len - 1, out.size());
    std::memcpy(buf, out.data(), n);
    buf[n] = 0;
    return out.size() < len ? MA_OK : MA_ERR_SHAPE;
}

void ma_plan_destroy(ma_plan_t* plan) { delete plan; }

int ma_profile_enable(int on) {
    g_prof_on = on != 0;
    return MA_OK;
}

int ma_profile_collect(double* ms_out, int64_t* launches_out, double* flops_out, double* bytes_out) {
    double ms[MA_PROF_CLASSES] = {0}, fl[MA_PROF_CLASSES] = {0}, by[MA_PROF_CLASSES] = {0};
    int64_t cnt[MA_PROF_CLASSES] = {0};
    int st = MA_OK;
    for (const ProfRec& r : g_prof_recs) {
        const auto& ev = g_prof_pool[r.ev];
        if (cudaEventSynchronize(ev.second) != cudaSuccess) {
            st = MA_ERR_CUDA;
            continue;
        }
        float t = 0.f;
        if (cudaEventElapsedTime(&t, ev.first, ev.second) != cudaSuccess) {
            st = MA_ERR_CUDA;
            continue;
        }
        ms[r.cls] += t;
        cnt[r.cls] += 1;
        fl[r.cls] += r.flops;
        by[r.cls] += r.bytes;
    }
    g_prof_recs.clear();
    for (int c = 0; c < MA_PROF_CLASSES; ++c) {
        if (ms_out) ms_out[c] = ms[c];
        if (launches_out) launches_out[c] = cnt[c];
        if (flops_out) flops_out[c] = fl[c];
        if (bytes_out) bytes_out[c] = by[c];
    }
    return st;
}

int ma_device_status(void* stream, int reset) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return MA_ERR_CUDA;
    if (reset) {
        const int z = 0;
        if (cudaMemcpyToSymbol(g_status, &z, sizeof(int)) != cudaSuccess) return MA_ERR_CUDA;
    }
    return v;
}

int ma_plan_status(ma_plan_t* plan, void* stream) {
    if (!plan) return MA_ERR_NULL;
    return ma_device_status(stream, 1);
}

int ma_device_status_async(int32_t* host_dst, void* stream) {
    if (!host_dst) return MA_ERR_NULL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MA_ERR_CUDA;
    return cudaMemcpyFromSymbolAsync(host_dst, g_status, sizeof(int32_t), 0, cudaMemcpyDeviceToHost,
                                     reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MA_OK
               : MA_ERR_CUDA;
}

int ma_set_wait_limit_ns(int64_t limit_ns) {
    if (limit_ns <= 0) return MA_ERR_ARG;
    g_host_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
    return MA_OK;
}

int ma_debug_build(void) {
#ifdef MA_DEBUG
    return 1;
#else
    return 0;
#endif
}

int ma_set_momentum_overlap(int on) {
    if (on != 0 && on != 1) return MA_ERR_ARG;
    g_momentum_overlap.store(on, std::memory_order_relaxed);
    return MA_OK;
}

int ma_selftest_wait_timeout(int64_t limit_ns, void* stream) {
    if (limit_ns <= 0 || limit_ns > 10000000000LL) return MA_ERR_ARG;
    int st = device_ok_and_sms(nullptr);
    if (st) return st;
    int* status = device_status_ptr();
    if (!status) return MA_ERR_CUDA;
    return launch_wait_selftest(limit_ns, status, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MA_OK
               : MA_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------- allocation-free Muon step
//
// For callers that cannot call cudaMalloc (see muonadamw.h): the scratch that
// muon_step_batched takes from the caller lives here, in one file-scope
// device array per GPU. The kernels and their order are exactly those of
// muon_step_batched; only the scratch base pointer differs.

static __device__ __align__(256) unsigned char g_noalloc_scratch[MA_STATIC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device, looked up once per
// device (host code only has a host-side stand-in for the symbol, which must
// never be handed to a kernel). NULL if the lookup fails. Host threads making
// their first call on a device at the same time are serialised by the cache.
static void* noalloc_scratch_ptr() {
    static ma::PerDevice<void*> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    void* ptr = nullptr;
    const cudaError_t e =
        cache.get(dev, &ptr, [](void** v) { return cudaGetSymbolAddress(v, g_noalloc_scratch); });
    return e == cudaSuccess ? ptr : nullptr;
}

extern "C" int muon_step_batched_noalloc(int batch, int64_t R, int64_t C, float* const* W, const void* const* G,
                                         int gdt, float* const* M, const ma_muon_hparams_t* hp, void* stream) {
    MuonGeom g;
    int st = check_muon_call(batch, R, C, W, G, gdt, M, hp, &g);
    if (st) return st;
    if (g.total == 0) return MA_OK;
    if (g.total > MA_STATIC_SCRATCH_BYTES) return MA_ERR_WORKSPACE;
    int sms = 0;
    if ((st = device_ok_and_sms(&sms))) return st;
    void* scratch = noalloc_scratch_ptr();
    if (!scratch) return MA_ERR_CUDA;
    int launches = 0;
    return run_muon(batch, g, W, G, gdt, M, *hp, scratch, reinterpret_cast<cudaStream_t>(stream), sms, &launches);
}
