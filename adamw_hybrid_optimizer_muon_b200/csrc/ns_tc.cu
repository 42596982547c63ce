// Newton-Schulz GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// One iteration of the odd polynomial ("MuonClip Optimizer",
// "Newton-Schulz Orthogonalization": X <- 1.5 X - 0.5 X (X^T X); in general
// X <- aX + b X(X^T X) + c X(X^T X)^2) runs on the short side of X, which is
// the same thing because X (X^T X) = (X X^T) X:
//
//   GRAM    A = X X^T             (m x m, symmetric; only tiles touching the
//                                  upper triangle are computed, and each one
//                                  writes its elements and their mirror)
//           epilogue: B = coef * A, coef = b * s^2 on the first iteration
//           (s = 1/(||u||_F + eps), the Frobenius normalisation), else b.
//   GRAMSQ  a symmetric m x m product out = b*Z + c*A Z (Z = A: b*A + c*A^2,
//           the extra term when c != 0; Z a second symmetric matrix that
//           commutes with A: the Gram-space chain's Q and A updates, which
//           reach X_N = Q_N X_0 from m x m products only); A Z = A Z^T by
//           symmetry, and only tiles touching the upper triangle run
//   APPLY   X' = s * (a X + B X)  (s only on the first iteration)
//   FINAL   the last APPLY. Its epilogue does the decoupled decay and the
//           update, W <- W*(1 - lr*wd) - lr*scale*X_N, straight into the
//           caller's fp32 weights, transposing back when the unit was tall.
//           X_N is never rounded or stored.
//
// Kernel structure: CTA pairs (clusters of 2), persistent over the 256 x 256
// output tiles of every unit of the launch's jobs (up to eight batches of
// one mode, tiles numbered job after job), 320 threads per CTA:
//   warp 0      TMA producer in each CTA: this CTA's half of the A tile
//               (128 rows x 64) and of the B tile (128 columns x 64), bf16,
//               128B swizzle, 6 stages of 32 KB (the final apply: 4, or 5 in
//               its deep variant for m >= 2048). Both
//               CTAs' loads complete on the leader CTA's stage barrier; there
//               is no multicast. A diagonal Gram tile loads only A.
//   warp 1      TMEM allocation in both CTAs (cta_group::2, 2 x 256 fp32
//               columns). In the leader only, MMA issue:
//               tcgen05.mma.cta_group::2.kind::f16, M = 256 (128 rows in each
//               CTA), N = 256, K = 16. Commits are multicast to both CTAs'
//               barriers: stage release and accumulator full.
//   warps 2..9  epilogue in both CTAs: each TMEM lane quadrant is read by two
//               warps, each taking half of the 256 columns, 32 at a time.
// Per unit of tile work, the pair moves (256 + 256) x 64 x 2 bytes from L2 for
// 256 x 256 x 64 multiply-adds: one third fewer bytes per flop than a
// single-CTA 128 x 256 tile. Units with m <= 128 would fill half of that tile;
// they run on a single-CTA instance of the same template (cta_group::1,
// 128 x 256 tiles, 128 x 128 for the Gram).
// B operand major-ness: for GRAM and GRAMSQ both operands are K-major rows
// (of the same matrix, or of A and Z). For APPLY the B operand is X itself,
// read MN-major (the contraction runs over X's rows), so no transposed copy
// is ever made.
// Tile order and L2: the applies walk each unit's tiles column by column, so
// the pairs running at the same time share a few column strips of X and all
// of the m x m Gram, which they load with an evict-last L2 policy; every
// bulk tensor store is evict-first (only the next launch reads it).
#include <climits>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace ma {

namespace {

#ifndef MA_NS_STAGES
#define MA_NS_STAGES 6
#endif
constexpr int BM = 256, BN = 256, BK = 64, STAGES = MA_NS_STAGES;
constexpr int HM = BM / 2, HN = BN / 2;                // rows of A / columns of B held by each CTA
constexpr uint32_t A_BYTES = HM * BK * 2;              // 16 KB
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 32 * (2 + EPI_WARPS);
// Epilogue staging: per epilogue warp one 32 x 32 bf16 block for the tile and
// one for its mirror (2 KB each, 64-byte rows, 64-byte swizzle), written out
// with bulk tensor stores.
constexpr uint32_t STG_BLOCK = 32 * 32 * 2;
// The epilogue warps wait for a whole tile's main loop; they sleep in the
// barrier wait rather than poll it (polling costs power, hence clock, on a
// power-capped part).
#ifndef MA_EPI_SLEEP_NS
#define MA_EPI_SLEEP_NS 20000
#endif
constexpr uint32_t kEpiSleepNs = MA_EPI_SLEEP_NS;
constexpr uint32_t STG_BYTES = EPI_WARPS * 2 * STG_BLOCK;  // 32 KB
// Final apply: each epilogue warp double-buffers a 32 x 32 fp32 block of W
// (128-byte rows) and, in the shallow variant, the matching 32 x 32 bf16
// block of X (64-byte rows). The 16-byte chunks of each row are XOR-swizzled
// by the row index, which keeps row-wise and column-wise accesses free of
// bank conflicts. Two variants share the code:
//  * shallow (DEEP = false): W and X staged, 96 KB, a 4-stage ring. For short
//    K loops (m < 2048), where the epilogue's latency is on the critical path
//    and the W stream nearly fills HBM;
//  * deep (DEEP = true): W staged, each lane reads its row of X straight from
//    global memory, 64 KB, a 5-stage ring. For m >= 2048, where the main loop
//    is long and more loads in flight keep the tensor pipe busier.
constexpr uint32_t WBUF = 32 * 128;                              // 4 KB
constexpr uint32_t XBUF = 32 * 64;                               // 2 KB
constexpr uint32_t fin_warp_bytes(bool deep) { return deep ? 2 * WBUF : 2 * WBUF + 2 * XBUF; }  // 8 / 12 KB
constexpr int kStages(int mode, bool deep) { return mode == NS_FINAL ? (deep ? 5 : 4) : STAGES; }
constexpr uint32_t kEpiBytes(int mode, bool deep) {
    return mode == NS_FINAL ? EPI_WARPS * fin_warp_bytes(deep) : STG_BYTES;
}
// Final-apply launches whose units all have at least this many rows (the K
// of the main loop) take the deep variant.
constexpr int kDeepFinalMinM = 2048;

constexpr int kMaxStages = 8;
// Wind-down after an abort: waits for the pair's own work in flight (issued
// MMAs, bulk loads) are bounded by at least this, whatever the wait limit.
constexpr long long kDrainNs = 50000000LL;

// Control block in shared memory, after the stage ring and the epilogue
// buffers. Its offsets are the same in both CTAs of a pair.
struct Ctl {
    uint64_t full[kMaxStages], empty[kMaxStages];  // stage ring: data landed / stage released by the MMAs
    uint64_t acc_full[2], acc_empty[2];            // TMEM accumulators: ready for the epilogue / free again
    uint64_t drain;                                // the MMA thread's last commit before an aborted exit
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t issued;                    // producer: stage uses armed and loaded so far
    int32_t consumed;                  // MMA thread: stage uses whose data it has waited for
    uint32_t stage_tx[kMaxStages];     // producer: bytes per CTA of the latest use of each stage
};
static_assert(sizeof(Ctl) <= 512, "control block");

// Tile shape of one kernel instance. PAIR: a CTA pair computes a 256 x 256
// tile (cta_group::2, each CTA holding 128 rows of A and 128 columns of B).
// Single CTA (for units with m <= 128, where a 256-row tile would be half
// empty): a 128-row tile, 256 columns for the applies and 128 for the Gram,
// cta_group::1.
template <int MODE, bool PAIR, bool DEEP = false>
struct Shape {
    static_assert(!DEEP || MODE == NS_FINAL, "only the final apply has a deep variant");
    static constexpr bool kApply = MODE == NS_APPLY || MODE == NS_FINAL;
    static constexpr int TM = PAIR ? BM : HM;                       // output tile rows
    static constexpr int TN = PAIR ? BN : (kApply ? BN : HN);       // output tile columns
    static constexpr int CN = PAIR ? TN / 2 : TN;                   // B columns staged by each CTA
    static constexpr uint32_t STAGE = A_BYTES + (uint32_t)CN * BK * 2;
    static constexpr uint32_t EPI = kEpiBytes(MODE, DEEP);
    static constexpr int FIT = (int)((232448u - EPI - 1536u) / STAGE);  // 227 KB of shared memory per CTA
    static constexpr int NST = PAIR ? kStages(MODE, DEEP) : (FIT < STAGES ? FIT : STAGES);
    static constexpr uint32_t TMEM = 2 * TN;                        // two fp32 accumulators
    static constexpr int CPW = TN / 64;                             // 32-column chunks per epilogue warp
    static constexpr size_t SMEM = (size_t)NST * STAGE + EPI + 1024 + 512;
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(NST <= kMaxStages, "stage ring");
};

struct TileCoord {
    int u, ti, tj;
};

// One job of a launch: a batch of same-shape units sharing this iteration's
// polynomial. A launch covers up to kMaxJobs jobs (same mode), so that small
// buckets fill the machine together.
constexpr int kMaxJobs = 8;
constexpr int kMaxW = 512;  // weight pointers over all jobs of a final-apply launch

struct NsJob {
    int32_t units, m, n, first;
    int64_t ldx, ldg, x_unit, g_unit;
    float a, b, c, coef_gram;
    const float* scale;
    const void* xin;
    const void* zin;    // GRAMSQ: the second operand Z (and the combine input); xin when it is A itself
    void* out;
    int32_t transposed, heads, cautious, w0;
    int32_t same;       // GRAM/GRAMSQ: both operands are rows of one matrix (a diagonal tile loads it once)
    int64_t Rh, C;
    float decay, lr_s, lr_wd;
    int32_t tiles_per_unit, mt, nt, kblocks, tile0;
};

struct NsLaunch {
    CUtensorMap mA[kMaxJobs], mB[kMaxJobs], mO[kMaxJobs];
    NsJob job[kMaxJobs];
    int32_t njobs, total_tiles;
    long long wait_limit_ns;
    int* status;
    float* W[kMaxW];
};

struct JobTile {
    int j;
    TileCoord tc;
};

// Tiles of one unit. GRAM/GRAMSQ: only the tiles (ti, tj) with ti <= tj, the
// ones that hold an element with row <= col, enumerated column by column.
__device__ __forceinline__ TileCoord decode_tile(int mode, int t, int tiles_per_unit, int mt, int nt) {
    TileCoord c;
    c.u = t / tiles_per_unit;
    int r = t - c.u * tiles_per_unit;
    if (mode == NS_GRAM || mode == NS_GRAMSQ) {
        int tj = 0;
        while (r >= tj + 1 && tj < nt - 1) {
            r -= tj + 1;
            ++tj;
        }
        c.ti = r;
        c.tj = tj;
    } else {
        // column by column: the pairs working at the same time share the few
        // column strips of X (the B operand) they read, and all of them read the
        // m x m Gram, the smaller operand when n > m
        c.tj = r / mt;
        c.ti = r - c.tj * mt;
    }
    return c;
}

// Global tile index of a launch -> (job, unit, tile row, tile column).
__device__ __forceinline__ JobTile decode_job_tile(const NsLaunch& L, int mode, int t) {
    JobTile r;
    int j = 0;
    while (j + 1 < L.njobs && t >= L.job[j + 1].tile0) ++j;
    const NsJob& J = L.job[j];
    r.j = j;
    r.tc = decode_tile(mode, t - J.tile0, J.tiles_per_unit, J.mt, J.nt);
    return r;
}

// o[t] = ca * in[t] + cv * v[t] for the 32 bf16 values in[0..31] of one row
// (zero where the row is out of range or t >= cols_left). o may alias v.
__device__ __forceinline__ void combine_row(const __nv_bfloat16* in, bool row_ok, int cols_left, float ca, float cv,
                                            const float (&v)[32], float (&o)[32]) {
    if (row_ok && cols_left >= 32) {
        const uint4* s = reinterpret_cast<const uint4*>(in);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 w = s[q];
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                o[8 * q + 2 * e] = ca * bf16_lo(wv[e]) + cv * v[8 * q + 2 * e];
                o[8 * q + 2 * e + 1] = ca * bf16_hi(wv[e]) + cv * v[8 * q + 2 * e + 1];
            }
        }
    } else {
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const float x = (row_ok && t < cols_left) ? __bfloat162float(in[t]) : 0.f;
            o[t] = ca * x + cv * v[t];
        }
    }
}

// This lane's 32 output values of one 32-column chunk (row `row`, columns
// col0..col0+31), before rounding: GRAM b*A (x s^2 on the first iteration),
// GRAMSQ b*A + c*A^2, APPLY/FINAL s*(a*X + B*X).
template <int MODE>
__device__ __forceinline__ void epilogue_values(const NsJob& p, const TileCoord& tc, int row, int col0, int* status,
                                                const float (&v)[32], float (&o)[32]) {  // o may alias v
    if (MODE == NS_GRAM) {
        float coef = p.coef_gram;
        if (p.first) {
            const float s = p.scale[tc.u];
            coef *= s * s;
        }
#pragma unroll
        for (int t = 0; t < 32; ++t) o[t] = coef * v[t];
    } else if (MODE == NS_GRAMSQ) {
        // acc = A Z^T (= A Z: both symmetric); out = b*Z + c*acc, Z read back 8 values at a time
        const int m = p.m;
        const float b = p.b, c = p.c;
        const __nv_bfloat16* Zin = reinterpret_cast<const __nv_bfloat16*>(p.zin) + (int64_t)tc.u * p.g_unit;
        const bool ok = row < m && MA_INB((int64_t)tc.u * p.g_unit + (int64_t)row * p.ldg + col0, min(32, m - col0),
                                          (int64_t)p.units * p.g_unit, status);
        combine_row(Zin + (int64_t)row * p.ldg + col0, ok, m - col0, b, c, v, o);
    } else {
        const int m = p.m, n = p.n;
        const float sa = p.first ? p.scale[tc.u] : 1.f;
        const __nv_bfloat16* Xin = reinterpret_cast<const __nv_bfloat16*>(p.xin) + (int64_t)tc.u * p.x_unit;
        const bool ok = row < m && MA_INB((int64_t)tc.u * p.x_unit + (int64_t)row * p.ldx + col0, min(32, n - col0),
                                          (int64_t)p.units * p.x_unit, status);
        combine_row(Xin + (int64_t)row * p.ldx + col0, ok, n - col0, sa * p.a, sa, v, o);
    }
}

// One weight: decoupled decay (optionally only where the update x and w agree in
// sign, the cautious reading), then the scaled orthogonalised update.
__device__ __forceinline__ float apply_update(float w, float x, float decay, float lrs, const NsJob& p) {
    if (p.cautious) return (x * w > 0.f ? w - p.lr_wd * w : w) - lrs * x;
    return w * decay - lrs * x;
}


// Byte offset of 16-byte chunk q of row r in a 64-byte-row block with the
// 64-byte swizzle that the bulk tensor store expects.
__device__ __forceinline__ uint32_t sw64(uint32_t r, uint32_t q) { return r * 64u + ((q ^ ((r >> 1) & 3u)) << 4); }

// Byte offset of 16-byte chunk q of row r in a 128-byte-row block of W.
__device__ __forceinline__ uint32_t sw128w(uint32_t r, uint32_t q) { return r * 128u + ((q ^ (r & 7u)) << 4); }

// Final apply: W <- W*(1 - lr*wd) - lr*scale*X_N in the caller's fp32 weights,
// run by each epilogue warp over its 32-column chunks of every tile.
//
// For each chunk, the 32 x 32 block of W (in W's own orientation: transposed
// back when the unit was tall) comes into shared memory by 16-byte
// asynchronous copies, and so does, in the shallow variant, the 32 x 32 block
// of X that the a*X term needs (none when a = 0). The first two chunks of a
// tile are fetched before the accumulator is ready, and each later chunk
// while the one before it is being computed, so the DRAM latency hides
// behind the main loop without holding registers. In the deep variant each
// lane reads the 32 values of its row of X straight from global memory, as
// the other epilogues read theirs. Each lane forms its row of X_N from the
// accumulator and X, updates its own row (or, transposed, its own column) of
// the W block in place, and the block goes back to W with coalesced 16-byte
// stores.
template <bool PAIR, bool DEEP>
__device__ __forceinline__ void final_epilogue(const NsLaunch& L, Ctl* ctl, int pair, int npairs, uint32_t rank,
                                               uint32_t tmem_base, int warp, int lane, uint8_t* wbuf,
                                               const AbortCtl& ab) {
    using S = Shape<NS_FINAL, PAIR, DEEP>;
    uint8_t* xbuf = wbuf + 2 * WBUF;  // shallow variant only
    constexpr int CPW = S::CPW;
    const int quad = warp & 3, half = (warp - 2) / 4;
    const long long limit = L.wait_limit_ns;
    const uint32_t acc_empty_leader0 = PAIR ? mapa_shared(smem_u32(&ctl->acc_empty[0]), 0) : 0u;
    const uint32_t acc_empty_leader1 = PAIR ? mapa_shared(smem_u32(&ctl->acc_empty[1]), 0) : 0u;
    int lt = 0;
    for (int t = pair; t < L.total_tiles; t += npairs, ++lt) {
        const JobTile jt = decode_job_tile(L, NS_FINAL, t);
        const NsJob& p = L.job[jt.j];
        const TileCoord tc = jt.tc;
        const int m = p.m, n = p.n;
        const float decay = p.decay, lrs = p.lr_s;
        const float sa = p.first ? p.scale[tc.u] : 1.f;
        const float ca = sa * p.a;
        const bool ax = p.a != 0.f;  // a = 0 (the Gram-space chain's X_N = s Q_N X_0): no X block needed
        const int acc = lt & 1;
        const uint32_t use = (uint32_t)(lt >> 1);
        const int row_lo = tc.ti * S::TM + (int)rank * HM + quad * 32;
        const int bidx = tc.u / p.heads, h = tc.u - bidx * p.heads;
        float* Wb = L.W[p.w0 + bidx] + (int64_t)h * p.Rh * p.C;
        const __nv_bfloat16* Xin = reinterpret_cast<const __nv_bfloat16*>(p.xin) + (int64_t)tc.u * p.x_unit;
        // element offsets and extents of this unit's W (in its matrix) and X (guarded build)
        const int64_t wbase = (int64_t)h * p.Rh * p.C, w_ext = (int64_t)p.heads * p.Rh * p.C;
        const int64_t xbase = (int64_t)tc.u * p.x_unit, x_ext = (int64_t)p.units * p.x_unit;
        (void)wbase; (void)w_ext; (void)xbase; (void)x_ext;
        // geometry of chunk c's W block: its first W row, first W column, and extents
        auto block = [&](int c, int& r0, int& c0, int& nr, int& rb) -> bool {
            const int col0 = tc.tj * S::TN + (half * CPW + c) * 32;
            if (row_lo >= m || col0 >= n) return false;
            if (!p.transposed) { r0 = row_lo; c0 = col0; nr = min(32, m - row_lo); rb = min(32, n - col0) * 4; }
            else { r0 = col0; c0 = row_lo; nr = min(32, n - col0); rb = min(32, m - row_lo) * 4; }
            return true;
        };
        auto fetch = [&](int c) {
            int r0, c0, nr, rb;
            if (c < CPW && block(c, r0, c0, nr, rb)) {
                uint8_t* buf = wbuf + (c & 1) * WBUF;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int row = 4 * i + (lane >> 3), q = lane & 7;
                    if (row < nr && q * 16 < rb &&
                        MA_INB(wbase + (int64_t)(r0 + row) * p.C + c0 + q * 4, 4, w_ext, L.status))
                        cp_async16(buf + sw128w(row, q), Wb + (int64_t)(r0 + row) * p.C + c0 + q * 4);
                }
                if (!DEEP && ax) {
                    // X rows row_lo.., columns col0..: 8 bf16 per copy; the row stride is a multiple of 8
                    const int col0 = tc.tj * S::TN + (half * CPW + c) * 32;
                    uint8_t* xb = xbuf + (c & 1) * XBUF;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int row = 8 * i + (lane >> 2), q = lane & 3;
                        if (row_lo + row < m && col0 + 8 * q < n &&
                            MA_INB(xbase + (int64_t)(row_lo + row) * p.ldx + col0 + 8 * q, 8, x_ext, L.status))
                            cp_async16(xb + sw64(row, q), Xin + (int64_t)(row_lo + row) * p.ldx + col0 + 8 * q);
                    }
                }
            }
            cp_async_commit();  // one group per chunk, empty or not, so the counts line up
        };
        fetch(0);
        fetch(1);
        int ok = 1;
        if (lane == 0)
            ok = mbar_wait_ctl(&ctl->acc_full[acc], use & 1u, ab, limit, L.status, kEpiSleepNs) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < CPW; ++c) {
            int r0, c0, nr, rb;
            if (!block(c, r0, c0, nr, rb)) break;  // warp-uniform
            uint8_t* buf = wbuf + (c & 1) * WBUF;
            // this lane's 32 values of X (row row_lo + lane), loaded before the accumulator
            // read; the row stride is a multiple of 8 and n - col0 of 8, so a group of 8
            // is wholly in range or out of it
            const int col0 = tc.tj * S::TN + (half * CPW + c) * 32;
            uint4 xv[4];
            if (DEEP && ax) {
                const bool xrow = row_lo + lane < m;
                const uint4* xs = reinterpret_cast<const uint4*>(Xin + (int64_t)(row_lo + lane) * p.ldx + col0);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    xv[q] = (xrow && col0 + 8 * q < n &&
                             MA_INB(xbase + (int64_t)(row_lo + lane) * p.ldx + col0 + 8 * q, 8, x_ext, L.status))
                                ? __ldg(xs + q)
                                : make_uint4(0u, 0u, 0u, 0u);
            }
            float o[32];
            tmem_ld32(tmem_base + (uint32_t)(acc * S::TN + (half * CPW + c) * 32) + ((uint32_t)(quad * 32) << 16), o);
            // chunk c's copies are the oldest group but one (chunk c + 1 was issued after it)
            cp_async_wait<1>();
            __syncwarp();
            if (!DEEP && ax) {
                const uint8_t* xb = xbuf + (c & 1) * XBUF;
#pragma unroll
                for (int q = 0; q < 4; ++q) xv[q] = *reinterpret_cast<const uint4*>(xb + sw64(lane, q));
            }
            // X_N row of this lane: s*(a*X + (B X)), s only on the first iteration
            if (ax) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t wv[4] = {xv[q].x, xv[q].y, xv[q].z, xv[q].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        o[8 * q + 2 * e] = ca * bf16_lo(wv[e]) + sa * o[8 * q + 2 * e];
                        o[8 * q + 2 * e + 1] = ca * bf16_hi(wv[e]) + sa * o[8 * q + 2 * e + 1];
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] *= sa;
            }
            if (!p.transposed) {
                // lane = row of W: 32 consecutive elements
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float4* wq = reinterpret_cast<float4*>(buf + sw128w(lane, q));
                    float4 w = *wq;
                    w.x = apply_update(w.x, o[4 * q + 0], decay, lrs, p);
                    w.y = apply_update(w.y, o[4 * q + 1], decay, lrs, p);
                    w.z = apply_update(w.z, o[4 * q + 2], decay, lrs, p);
                    w.w = apply_update(w.w, o[4 * q + 3], decay, lrs, p);
                    *wq = w;
                }
            } else {
                // lane = column of W: element t of the lane's X_N row is W[t][lane]
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    float* wq = reinterpret_cast<float*>(buf + sw128w(q, lane >> 2) + (lane & 3) * 4);
                    *wq = apply_update(*wq, o[q], decay, lrs, p);
                }
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int row = 4 * i + (lane >> 3), q = lane & 7;
                // streaming stores (evict-first in L2): the updated weights are not
                // read again in this launch, unlike the Gram and X strips
                if (row < nr && q * 16 < rb &&
                    MA_INB(wbase + (int64_t)(r0 + row) * p.C + c0 + q * 4, 4, w_ext, L.status))
                    __stcs(reinterpret_cast<float4*>(Wb + (int64_t)(r0 + row) * p.C + c0 + q * 4),
                           *reinterpret_cast<const float4*>(buf + sw128w(row, q)));
            }
            __syncwarp();  // both buffers of chunk c are free again
            fetch(c + 2);
        }
        cp_async_wait<0>();  // drop the copies of chunks this tile does not use
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            if (PAIR) mbar_arrive_cluster(acc ? acc_empty_leader1 : acc_empty_leader0);
            else mbar_arrive(&ctl->acc_empty[acc]);
        }
    }
    cp_async_wait<0>();
}

// After an abort, with every role of both CTAs stopped (no thread issues
// anything more), the leader's MMA thread waits for the pair's work in
// flight, bounded by the drain limit but not cut short by the abort:
//  * every MMA it issued (one more commit, on the drain barrier);
//  * every bulk load either producer issued that the MMAs never consumed.
//    Each such stage use has at most one outstanding phase. Where both
//    producers issued it, the phase completes when the bytes land. Where only
//    the leader did (it armed the barrier for both CTAs' bytes), the peer's
//    missing bytes are completed by hand; where only the peer did (the leader
//    never armed it), the leader arms it for the peer's bytes. Either way the
//    phase then completes exactly when the issued copies have landed.
// Returns normally in every case; a drain wait that runs out records
// MA_ERR_TIMEOUT like any other wait.
template <int NST, bool PAIR>
__device__ __forceinline__ void abort_drain(Ctl* ctl, const AbortCtl& ab, const NsLaunch& L) {
    const long long lim = L.wait_limit_ns > kDrainNs ? L.wait_limit_ns : kDrainNs;
    if (PAIR) tc_commit_pair(&ctl->drain);
    else tc_commit(&ctl->drain);
    mbar_wait_ctl(&ctl->drain, 0, ab, lim, L.status, 0, false, true);
    const int consumed = ctl->consumed;
    const int own = ctl->issued;
    const int peer = PAIR ? ld_cluster_s32(mapa_shared(smem_u32(&ctl->issued), 1)) : own;
    const int last = own > peer ? own : peer;
    for (int u = consumed; u < last; ++u) {
        const int st = u % NST;
        const uint32_t par = (uint32_t)(u / NST) & 1u;
        const bool mine = u < own, theirs = u < peer;
        if (PAIR && mine && !theirs) {
            mbar_complete_tx(&ctl->full[st], ctl->stage_tx[st]);
        } else if (PAIR && theirs && !mine) {
            const uint32_t tx = (uint32_t)ld_cluster_s32(mapa_shared(smem_u32(&ctl->stage_tx[st]), 1));
            mbar_arrive_expect_tx(&ctl->full[st], tx);
        }
        mbar_wait_ctl(&ctl->full[st], par, ab, lim, L.status, 0, PAIR, true);
    }
}

template <int MODE, bool PAIR, bool DEEP = false>
__global__ void __launch_bounds__(THREADS, 1)
    ns_tc_kernel(const __grid_constant__ NsLaunch L) {
    using S = Shape<MODE, PAIR, DEEP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int NST = S::NST;
    uint8_t* staging = smem + NST * S::STAGE;
    Ctl* ctl = reinterpret_cast<Ctl*>(staging + S::EPI);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    griddep_launch_dependents();
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0 = leader of the pair
    const bool leader = rank == 0;
    const int pair = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;
    const int npairs = PAIR ? (int)cluster_count_x() : (int)gridDim.x;
    const int total_tiles = L.total_tiles;
    const long long limit = L.wait_limit_ns;
    constexpr bool kApply = (MODE == NS_APPLY || MODE == NS_FINAL);
    const AbortCtl ab{&ctl->abort_flag, PAIR ? mapa_shared(smem_u32(&ctl->abort_flag), rank ^ 1u) : 0u};

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&ctl->full[s], 1);   // leader: its own arrive.expect_tx + both CTAs' bytes
            mbar_init(&ctl->empty[s], 1);  // both: one multicast commit per use
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ctl->acc_full[a], 1);                              // both: one multicast commit per tile
            mbar_init(&ctl->acc_empty[a], (PAIR ? 2 : 1) * EPI_WARPS);  // leader: every epilogue warp of the pair
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort_flag = 0;
        ctl->issued = 0;
        ctl->consumed = 0;
        fence_barrier_init();
        for (int j = 0; j < L.njobs; ++j) {
            prefetch_tensormap(&L.mA[j]);
            prefetch_tensormap(&L.mB[j]);
            if (MODE != NS_FINAL) prefetch_tensormap(&L.mO[j]);
        }
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(&ctl->tmem_base, S::TMEM);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&ctl->tmem_base, S::TMEM);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if (PAIR) cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated in both
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    griddep_wait();  // the previous kernel's results (and its reads of our outputs) are complete

    if (warp == 0) {
        if (lane == 0) {
            // In the applies every pair working at the same time reads all of
            // the m x m Gram (the A operand), one wave after another: keep it in
            // L2 ahead of the X strips, which each wave reads once.
            const uint64_t keep = l2_evict_last_policy();
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int t = pair; t < total_tiles && ok; t += npairs) {
                const JobTile jt = decode_job_tile(L, MODE, t);
                const TileCoord tc = jt.tc;
                const CUtensorMap* mapA = &L.mA[jt.j];
                const CUtensorMap* mapB = &L.mB[jt.j];
                const int kblocks = L.job[jt.j].kblocks;
                const int arow = tc.ti * S::TM + (int)rank * HM;
                const int bcol = tc.tj * S::TN + (int)rank * S::CN;
                // a diagonal Gram tile multiplies a block of rows by itself: B is A's smem
                const bool diag = !kApply && tc.ti == tc.tj && L.job[jt.j].same;
                const uint32_t stage_tx = diag ? A_BYTES : S::STAGE;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_ctl(&ctl->empty[stage], phase ^ 1u, ab, limit, L.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + stage * S::STAGE;
                    uint8_t* sb = sa + A_BYTES;
                    if (PAIR) {
                        if (leader) mbar_arrive_expect_tx(&ctl->full[stage], 2 * stage_tx);
                        const uint32_t fb = mapa_shared(smem_u32(&ctl->full[stage]), 0);
                        if (kApply) tma_load_3d_pair_hint(sa, mapA, fb, kb * BK, arow, tc.u, keep);
                        else tma_load_3d_pair(sa, mapA, fb, kb * BK, arow, tc.u);
                        if (!kApply) {
                            if (!diag) tma_load_3d_pair(sb, mapB, fb, kb * BK, bcol, tc.u);
                        } else {
#pragma unroll
                            for (int q = 0; q < S::CN / 64; ++q)
                                tma_load_3d_pair(sb + q * (64 * BK * 2), mapB, fb, bcol + q * 64, kb * BK, tc.u);
                        }
                    } else {
                        mbar_arrive_expect_tx(&ctl->full[stage], stage_tx);
                        if (kApply) tma_load_3d_hint(sa, mapA, &ctl->full[stage], kb * BK, arow, tc.u, keep);
                        else tma_load_3d(sa, mapA, &ctl->full[stage], kb * BK, arow, tc.u);
                        if (!kApply) {
                            if (!diag) tma_load_3d(sb, mapB, &ctl->full[stage], kb * BK, bcol, tc.u);  // CN = 128 rows
                        } else {
#pragma unroll
                            for (int q = 0; q < S::CN / 64; ++q)
                                tma_load_3d(sb + q * (64 * BK * 2), mapB, &ctl->full[stage], bcol + q * 64, kb * BK,
                                            tc.u);
                        }
                    }
                    // what the abort drain needs: this use is armed (leader) and its loads issued
                    ctl->stage_tx[stage] = stage_tx;
                    ctl->issued = ++issued;
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Tail: wait until the MMAs have released every stage this CTA filled,
            // so that no commit arrives on this CTA's barriers after it exits.
            for (int i = 0; i < NST && ok; ++i) {
                ok = mbar_wait_ctl(&ctl->empty[stage], phase ^ 1u, ab, limit, L.status);
                if (++stage == NST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            constexpr uint32_t IDESC = idesc_bf16_f32(S::TM, S::TN, kApply ? 1 : 0);
            int stage = 0;
            uint32_t phase = 0;
            int consumed = 0;
            bool ok = true;
            int lt = 0;
            for (int t = pair; t < total_tiles && ok; t += npairs, ++lt) {
                const int acc = lt & 1;
                const uint32_t use = (uint32_t)(lt >> 1);
                if (!mbar_wait_ctl(&ctl->acc_empty[acc], (use & 1u) ^ 1u, ab, limit, L.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * S::TN);
                const JobTile jt = decode_job_tile(L, MODE, t);
                const int kblocks = L.job[jt.j].kblocks;
                const bool diag = !kApply && jt.tc.ti == jt.tc.tj && L.job[jt.j].same;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_ctl(&ctl->full[stage], phase, ab, limit, L.status)) {
                        ok = false;
                        break;
                    }
                    ctl->consumed = ++consumed;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + stage * S::STAGE);
                    const uint32_t b0 = diag ? a0 : a0 + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(a0 + kk * 32, 16, 1024);
                        uint64_t bdesc;
                        if (kApply)
                            bdesc = smem_desc_sw128(b0 + kk * (16 * 128), 64 * BK * 2, 1024);
                        else
                            bdesc = smem_desc_sw128(b0 + kk * 32, 16, 1024);
                        if (PAIR) tc_mma_f16_pair(d_tmem, adesc, bdesc, IDESC, (kb | kk) != 0 ? 1u : 0u);
                        else tc_mma_f16(d_tmem, adesc, bdesc, IDESC, (kb | kk) != 0 ? 1u : 0u);
                    }
                    if (PAIR) tc_commit_pair_mc(&ctl->empty[stage], 0x3);
                    else tc_commit(&ctl->empty[stage]);
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (PAIR) tc_commit_pair_mc(&ctl->acc_full[acc], 0x3);
                else tc_commit(&ctl->acc_full[acc]);
            }
        }
    } else if (MODE == NS_FINAL) {
        final_epilogue<PAIR, DEEP>(L, ctl, pair, npairs, rank, tmem_base, warp, lane,
                                   staging + (warp - 2) * fin_warp_bytes(DEEP), ab);
    } else {
        const int quad = warp & 3;              // TMEM lanes [32*quad, 32*quad + 32)
        const int half = (warp - 2) / 4;        // which half of the 256 columns
        uint8_t* stg = staging + (warp - 2) * 2 * STG_BLOCK;
        // outputs are read only by the next launch, long after L2 has turned over
        const uint64_t stream_out = l2_evict_first_policy();
        const uint32_t acc_empty_leader0 = PAIR ? mapa_shared(smem_u32(&ctl->acc_empty[0]), 0) : 0u;
        const uint32_t acc_empty_leader1 = PAIR ? mapa_shared(smem_u32(&ctl->acc_empty[1]), 0) : 0u;
        int lt = 0;
        for (int t = pair; t < total_tiles; t += npairs, ++lt) {
            const JobTile jt = decode_job_tile(L, MODE, t);
            const NsJob& p = L.job[jt.j];
            const CUtensorMap* mapOut = &L.mO[jt.j];
            const TileCoord tc = jt.tc;
            const int acc = lt & 1;
            const uint32_t use = (uint32_t)(lt >> 1);
            const int row_lo = tc.ti * S::TM + (int)rank * HM + quad * 32;
            const int row = row_lo + lane;
            int ok = 1;
            if (lane == 0)
                ok = mbar_wait_ctl(&ctl->acc_full[acc], use & 1u, ab, limit, L.status, kEpiSleepNs) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const int limit_cols = kApply ? p.n : p.m;
#pragma unroll 1
            for (int c = 0; c < S::CPW; ++c) {
                const int cc = half * S::CPW + c;
                const int col0 = tc.tj * S::TN + cc * 32;
                if (col0 >= limit_cols || row_lo >= p.m) break;                  // warp-uniform
                if (!kApply && col0 < row_lo) continue;                          // below the diagonal
                float o[32];
                tmem_ld32(tmem_base + (uint32_t)(acc * S::TN + cc * 32) + ((uint32_t)(quad * 32) << 16), o);
                epilogue_values<MODE>(p, tc, row, col0, L.status, o, o);  // in place
                // Stage this warp's 32 x 32 block (and, for an off-diagonal Gram
                // chunk, its transpose), then write both with bulk tensor stores:
                // each leaves shared memory as contiguous 64-byte rows.
                const bool mirror = !kApply && col0 > row_lo;
                if (lane == 0) bulk_wait_group_read0();  // the previous chunk's stores have read their source
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 w;
                    w.x = pack_bf16x2(o[8 * q + 0], o[8 * q + 1]);
                    w.y = pack_bf16x2(o[8 * q + 2], o[8 * q + 3]);
                    w.z = pack_bf16x2(o[8 * q + 4], o[8 * q + 5]);
                    w.w = pack_bf16x2(o[8 * q + 6], o[8 * q + 7]);
                    *reinterpret_cast<uint4*>(stg + sw64(lane, q)) = w;
                }
                if (mirror) {
                    const uint32_t lo = ((uint32_t)lane & 7u) << 1, qq = (uint32_t)lane >> 3;
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        *reinterpret_cast<__nv_bfloat16*>(stg + STG_BLOCK + sw64(t, qq) + lo) = __float2bfloat16_rn(o[t]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d_hint(mapOut, stg, col0, row_lo, tc.u, stream_out);
                    if (mirror) tma_store_3d_hint(mapOut, stg + STG_BLOCK, row_lo, col0, tc.u, stream_out);
                    bulk_commit_group();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR) mbar_arrive_cluster(acc ? acc_empty_leader1 : acc_empty_leader0);
                else mbar_arrive(&ctl->acc_empty[acc]);
            }
        }
        if (lane == 0) bulk_wait_group0();  // every bulk store of this warp has completed
    }

    // Every role of this CTA has stopped issuing; wait for the peer's too. The
    // normal path is drained by construction (the producers waited for the
    // MMAs to release their stages, the epilogues for every accumulator).
    // After an abort, which reached both CTAs before this barrier, the leader
    // drains the pair's MMAs and bulk loads before either CTA releases TMEM
    // or exits.
    __syncwarp();
    __syncthreads();
    tc_fence_before();
    if (PAIR) cluster_sync_all();
    if (ctl->abort_flag && leader && warp == 1 && lane == 0) abort_drain<NST, PAIR>(ctl, ab, L);
    __syncwarp();
    __syncthreads();
    tc_fence_before();
    if (PAIR) cluster_sync_all();  // neither CTA leaves while the pair may still touch its memory
    if (warp == 1) {
        tc_fence_after();
        if (PAIR) tmem_dealloc_pair(tmem_base, S::TMEM);
        else tmem_dealloc(tmem_base, S::TMEM);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (thread-safe static
// initialisation); NULL when the driver does not provide it.
EncodeTiledFn encode_fn() {
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

// 3-D bf16 map over [units][rows][inner] with row stride `ld` and unit stride
// `unit` (elements), zero fill out of bounds (loads) / clipping (stores).
bool make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t units, uint64_t ld,
              uint64_t unit, uint32_t box_inner, uint32_t box_rows,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {inner, rows, units};
    cuuint64_t strides[2] = {ld * 2, unit * 2};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Once per device and kernel instance: allow its dynamic shared memory and
// find how many pairs (or CTAs) can be resident at once. Not legal inside a
// stream capture the first time; ns_tc_setup runs it for every instance.
// Concurrent first calls from several host threads are serialised per
// instance, and a launch never sees a device whose attribute is not yet set.
template <int MODE, bool PAIR, bool DEEP = false>
cudaError_t setup_mode(int num_sms, int* max_units_out) {
    using S = Shape<MODE, PAIR, DEEP>;
    static PerDevice<int> cache;  // resident pairs (or CTAs) per device, once its attributes are set
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    return cache.get(dev, max_units_out, [num_sms](int* max_units) -> cudaError_t {
        cudaError_t e =
            cudaFuncSetAttribute(ns_tc_kernel<MODE, PAIR, DEEP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)S::SMEM);
        if (e != cudaSuccess) return e;
        if (PAIR) {
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cudaLaunchConfig_t qc = {};
            qc.gridDim = dim3(2 * (unsigned)(num_sms / 2));
            qc.blockDim = dim3(THREADS);
            qc.dynamicSmemBytes = S::SMEM;
            qc.attrs = attr;
            qc.numAttrs = 1;
            int nclusters = 0;
            e = cudaOccupancyMaxActiveClusters(&nclusters, ns_tc_kernel<MODE, PAIR, DEEP>, &qc);
            if (e != cudaSuccess) return e;
            if (nclusters < 1) return cudaErrorInvalidConfiguration;
            *max_units = nclusters;
        } else {
            int per_sm = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ns_tc_kernel<MODE, PAIR, DEEP>, THREADS,
                                                              S::SMEM);
            if (e != cudaSuccess) return e;
            if (per_sm < 1) return cudaErrorInvalidConfiguration;
            *max_units = per_sm * num_sms;
        }
        return cudaSuccess;
    });
}

template <int MODE, bool PAIR, bool DEEP = false>
cudaError_t launch_mode(const NsJobIn* jobs, int njobs, int num_sms, cudaStream_t s) {
    using S = Shape<MODE, PAIR, DEEP>;
    if (njobs < 1 || njobs > kMaxJobs) return cudaErrorInvalidValue;
    static thread_local NsLaunch L;  // ~9 KB parameter block, copied at launch
    std::memset(&L, 0, sizeof(L));
    int tile0 = 0, w0 = 0;
    for (int j = 0; j < njobs; ++j) {
        const NsParams& p = *jobs[j].p;
        const void* x_buf = jobs[j].x_buf;
        const void* g_buf = jobs[j].g_buf;
        NsJob& J = L.job[j];
        int kblocks, mt, nt, tiles;
        mt = (p.m + S::TM - 1) / S::TM;
        if (MODE == NS_GRAM || MODE == NS_GRAMSQ) {
            nt = (p.m + S::TN - 1) / S::TN;  // S::TN == S::TM for the Gram
            tiles = nt * (nt + 1) / 2;
            if (MODE == NS_GRAM) {
                kblocks = (p.n + BK - 1) / BK;
                if (!make_map(&L.mA[j], x_buf, p.n, p.m, p.units, p.ldx, p.x_unit, BK, HM)) return cudaErrorInvalidValue;
            } else {
                kblocks = (p.m + BK - 1) / BK;
                if (!make_map(&L.mA[j], p.xin, p.m, p.m, p.units, p.ldg, p.g_unit, BK, HM))
                    return cudaErrorInvalidValue;
            }
            // both operands are 128-row, 64-deep K-major boxes: of the same matrix,
            // or (GRAMSQ with a second operand) of Z
            if (MODE == NS_GRAMSQ && p.zin && p.zin != p.xin) {
                if (!make_map(&L.mB[j], p.zin, p.m, p.m, p.units, p.ldg, p.g_unit, BK, HM))
                    return cudaErrorInvalidValue;
                J.same = 0;
            } else {
                L.mB[j] = L.mA[j];
                J.same = 1;
            }
            if (!make_map(&L.mO[j], p.out, p.m, p.m, p.units, p.ldg, p.g_unit, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
                return cudaErrorInvalidValue;
        } else {
            nt = (p.n + S::TN - 1) / S::TN;
            tiles = mt * nt;
            kblocks = (p.m + BK - 1) / BK;
            if (!make_map(&L.mA[j], g_buf, p.m, p.m, p.units, p.ldg, p.g_unit, BK, HM)) return cudaErrorInvalidValue;
            if (!make_map(&L.mB[j], x_buf, p.n, p.m, p.units, p.ldx, p.x_unit, 64, BK)) return cudaErrorInvalidValue;
            if (MODE == NS_APPLY &&
                !make_map(&L.mO[j], p.out, p.n, p.m, p.units, p.ldx, p.x_unit, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
                return cudaErrorInvalidValue;
        }
        J.units = p.units; J.m = p.m; J.n = p.n; J.first = p.first;
        J.ldx = p.ldx; J.ldg = p.ldg; J.x_unit = p.x_unit; J.g_unit = p.g_unit;
        J.a = p.a; J.b = p.b; J.c = p.c; J.coef_gram = p.coef_gram;
        J.scale = p.scale; J.xin = p.xin; J.out = p.out;
        J.zin = (MODE == NS_GRAMSQ && p.zin) ? p.zin : p.xin;
        J.transposed = p.transposed; J.heads = p.heads; J.cautious = p.cautious;
        J.Rh = p.Rh; J.C = p.C; J.decay = p.decay; J.lr_s = p.lr_s; J.lr_wd = p.lr_wd;
        J.tiles_per_unit = tiles; J.mt = mt; J.nt = nt; J.kblocks = kblocks;
        J.tile0 = tile0;
        J.w0 = w0;
        if (MODE == NS_FINAL) {
            const int batch = p.heads > 0 ? p.units / p.heads : 0;
            if (w0 + batch > kMaxW) return cudaErrorInvalidValue;
            for (int b = 0; b < batch; ++b) L.W[w0 + b] = p.W[b];
            w0 += batch;
        }
        const long long t = (long long)tile0 + (long long)tiles * p.units;
        if (t > INT_MAX) return cudaErrorInvalidValue;
        tile0 = (int)t;
    }
    L.njobs = njobs;
    L.total_tiles = tile0;
    L.wait_limit_ns = jobs[0].p->wait_limit_ns;
    L.status = jobs[0].p->status;
    if (tile0 <= 0) return cudaSuccess;
    int max_units = 0;
    cudaError_t e = setup_mode<MODE, PAIR, DEEP>(num_sms, &max_units);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = MA_PDL;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    const long long units = tile0 < max_units ? tile0 : max_units;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((PAIR ? 2 : 1) * units));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = S::SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = PAIR ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, ns_tc_kernel<MODE, PAIR, DEEP>, L);
}

// Units with m <= 128 fill only half of a pair's 256-row tile: they take the
// single-CTA kernel.
bool single_cta(const NsParams& p) { return p.m <= HM; }

template <int MODE>
cudaError_t launch_split(const NsJobIn* jobs, int njobs, int num_sms, cudaStream_t s, int* launched) {
    NsJobIn big[kMaxJobs], small[kMaxJobs];
    int nb = 0, ns = 0;
    for (int j = 0; j < njobs && j < kMaxJobs; ++j) {
        if (single_cta(*jobs[j].p)) small[ns++] = jobs[j];
        else big[nb++] = jobs[j];
    }
    if (njobs > kMaxJobs) return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (nb > 0) {
        // the final apply takes its deep variant when every unit's K loop is long
        bool deep = MODE == NS_FINAL;
        for (int j = 0; j < nb; ++j) deep = deep && big[j].p->m >= kDeepFinalMinM;
        if (MODE == NS_FINAL && deep) e = launch_mode<NS_FINAL, true, true>(big, nb, num_sms, s);
        else e = launch_mode<MODE, true>(big, nb, num_sms, s);
        if (e != cudaSuccess) return e;
        ++*launched;
    }
    if (ns > 0) {
        e = launch_mode<MODE, false>(small, ns, num_sms, s);
        if (e != cudaSuccess) return e;
        ++*launched;
    }
    return cudaSuccess;
}

// Q = a*I + b*A for every unit: the first factor of the Gram-space chain.
// One warp per row of a unit (grid-stride over units x rows); lanes take the
// row's 16-byte groups of eight bf16 values, four groups in flight at a time.
__device__ __forceinline__ uint4 q1_group(uint4 v, int row, int c0, float a, float b) {
    const uint32_t x[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = b * bf16_lo(x[e]);
        f[2 * e + 1] = b * bf16_hi(x[e]);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e)
        if (row == c0 + e) f[e] += a;
    uint4 o;
    o.x = pack_bf16x2(f[0], f[1]);
    o.y = pack_bf16x2(f[2], f[3]);
    o.z = pack_bf16x2(f[4], f[5]);
    o.w = pack_bf16x2(f[6], f[7]);
    return o;
}

__global__ void __launch_bounds__(256) ns_q1_kernel(const __nv_bfloat16* __restrict__ A, __nv_bfloat16* __restrict__ Q,
                                                    int m, int64_t ldg, int64_t g_unit, int units, float a, float b,
                                                    int* status) {
    griddep_launch_dependents();
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)units * m;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x / 32);
    const int full = m / 8;  // whole 16-byte groups in a row (the row stride is a multiple of 8)
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); r < rows; r += nwarps) {
        const int64_t u = r / m;
        const int row = (int)(r - u * m);
        const int64_t off = u * g_unit + (int64_t)row * ldg;
        const uint4* src = reinterpret_cast<const uint4*>(A + off);
        uint4* dst = reinterpret_cast<uint4*>(Q + off);
        const int64_t ext = (int64_t)units * g_unit;  // elements of A and of Q (guarded build)
        (void)ext;
        int q = lane;
        for (; q + 96 < full; q += 128) {
            if (!MA_INB(off + 8 * q, 8 * 97, ext, status)) break;  // groups q .. q + 96
            uint4 v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = __ldcs(src + q + 32 * k);
#pragma unroll
            for (int k = 0; k < 4; ++k) __stcs(dst + q + 32 * k, q1_group(v[k], row, 8 * (q + 32 * k), a, b));
        }
        for (; q < full; q += 32)
            if (MA_INB(off + 8 * q, 8, ext, status)) __stcs(dst + q, q1_group(__ldcs(src + q), row, 8 * q, a, b));
        if (lane == 0 && MA_INB(off, m, ext, status)) {
            for (int c = 8 * full; c < m; ++c) {
                const float f = b * __bfloat162float(A[off + c]) + (row == c ? a : 0.f);
                Q[off + c] = __float2bfloat16_rn(f);
            }
        }
    }
}

}  // namespace

cudaError_t launch_ns_q1(const void* A, void* Q, int m, int64_t ldg, int64_t g_unit, int units, float a, float b,
                         int* status, int num_sms, cudaStream_t s) {
    if (units <= 0 || m <= 0) return cudaSuccess;
    const int64_t rows = (int64_t)units * m;
    int64_t blocks = (rows + 7) / 8;  // eight warps a block, one row each
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    return launch_pdl(ns_q1_kernel, dim3((unsigned)blocks), dim3(256), 0, s,
                      reinterpret_cast<const __nv_bfloat16*>(A), reinterpret_cast<__nv_bfloat16*>(Q), m, ldg, g_unit,
                      units, a, b, status);
}

size_t ns_tc_smem_bytes() {  // the largest dynamic shared memory of any instance
    size_t m = 0;
#define MA_MAXS(M, P) m = Shape<M, P>::SMEM > m ? Shape<M, P>::SMEM : m;
    MA_MAXS(NS_GRAM, true) MA_MAXS(NS_GRAM, false) MA_MAXS(NS_GRAMSQ, true) MA_MAXS(NS_GRAMSQ, false)
    MA_MAXS(NS_APPLY, true) MA_MAXS(NS_APPLY, false) MA_MAXS(NS_FINAL, true) MA_MAXS(NS_FINAL, false)
    m = Shape<NS_FINAL, true, true>::SMEM > m ? Shape<NS_FINAL, true, true>::SMEM : m;
#undef MA_MAXS
    return m;
}

cudaError_t ns_tc_setup(int num_sms) {
    if (!encode_fn()) return cudaErrorNotSupported;
    int u = 0;
    cudaError_t e;
#define MA_SETUP(M, P) \
    if ((e = setup_mode<M, P>(num_sms, &u)) != cudaSuccess) return e;
    MA_SETUP(NS_GRAM, true) MA_SETUP(NS_GRAM, false) MA_SETUP(NS_GRAMSQ, true) MA_SETUP(NS_GRAMSQ, false)
    MA_SETUP(NS_APPLY, true) MA_SETUP(NS_APPLY, false) MA_SETUP(NS_FINAL, true) MA_SETUP(NS_FINAL, false)
    if ((e = setup_mode<NS_FINAL, true, true>(num_sms, &u)) != cudaSuccess) return e;
#undef MA_SETUP
    return cudaSuccess;
}

bool ns_tc_is_final(const void* func) {
    return func == reinterpret_cast<const void*>(ns_tc_kernel<NS_FINAL, true>) ||
           func == reinterpret_cast<const void*>(ns_tc_kernel<NS_FINAL, true, true>) ||
           func == reinterpret_cast<const void*>(ns_tc_kernel<NS_FINAL, false>);
}

size_t ns_tc_launch_bytes() { return sizeof(NsLaunch); }

int ns_tc_patch_final(void* launch, NsFinalPatchFn f, void* ctx) {
    NsLaunch* L = reinterpret_cast<NsLaunch*>(launch);
    for (int j = 0; j < L->njobs; ++j) {
        NsJob& J = L->job[j];
        const int st = f(ctx, L->W[J.w0], J.Rh, J.C, &J.decay, &J.lr_s, &J.lr_wd);
        if (st) return st;
    }
    return 0;
}
int ns_tc_max_jobs() { return kMaxJobs; }
int ns_tc_max_weights() { return kMaxW; }

cudaError_t launch_ns_tc_group(int mode, const NsJobIn* jobs, int njobs, int num_sms, cudaStream_t s,
                               int* launched) {
    int dummy = 0;
    if (!launched) launched = &dummy;
    switch (mode) {
        case NS_GRAM: return launch_split<NS_GRAM>(jobs, njobs, num_sms, s, launched);
        case NS_GRAMSQ: return launch_split<NS_GRAMSQ>(jobs, njobs, num_sms, s, launched);
        case NS_APPLY: return launch_split<NS_APPLY>(jobs, njobs, num_sms, s, launched);
        case NS_FINAL: return launch_split<NS_FINAL>(jobs, njobs, num_sms, s, launched);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_ns_tc(int mode, const NsParams& p, const void* x_buf, const void* g_buf, int num_sms,
                         cudaStream_t s) {
    NsJobIn j{&p, x_buf, g_buf};
    return launch_ns_tc_group(mode, &j, 1, num_sms, s, nullptr);
}

}  // namespace ma
