// Tensor-core band sweeps for bf16 storage (sm_100a: TMA + tcgen05 + TMEM).
//
// Same sweeps and epilogues as the SIMT kernels (see simt_sweep.cuh), with
// the band contractions on the 5th-generation tensor cores:
//   S  = A_blk B_chunk^T   128 x 128 x 64, bf16 in, fp32 accumulation in TMEM
//   G  = A2_blk B2_chunk^T (dS sweeps only)
//   O += P X_chunk         128 x 64 x 128, P (or dS) rounded to bf16 and stored
//                          in TMEM (two bf16 per column, the contraction's A
//                          operand), X read MN-major straight from its TMA tile.
// One CTA owns a block of 128 rows (TMEM lanes) of one (batch, head) problem
// and walks the band's column chunks [r0 - W, r0 + 127 + W] in steps of 128.
//
// Warp roles:
//   NEPI epilogue warps (16 for PV, 8 for the others): warp w reads TMEM lanes
//              32*(w%4)..+31 (its rows) and a 128/(NEPI/4)-column part of each
//              chunk;
//   a loader:  TMA tiles (lane 0) and the chunk's column vectors (all lanes)
//              into a ring of NST stages;
//   a score-MMA issuer, and for PV and dS a second issuer for P X (one
//              elected lane each).
// Pipelines are mbarriers; every wait is bounded and a timeout records
// SA_ERR_TIMEOUT in the status word and unwinds.
//
// Dual updates use the previous value of the updated dual as the exponent
// shift (u_new = u_old - log sum_j exp(S + u_old + v)): every term is then a
// plan entry of a plan with unit columns (or rows) and is at most 1.  The
// first row update of a solve (no previous u) uses an online max instead.
#pragma once

#include "common.cuh"
#include "simt_sweep.cuh"
#include "tc_ptx.cuh"

namespace sa {
namespace tcs {

using simt::SweepArgs;
using simt::MAXT;
constexpr int LSE = simt::LSE, WSUM = simt::WSUM, PV = simt::PV, DS1 = simt::DS1,
              DSD = simt::DSD;
// The modes this kernel runs: the first (online) dual update of a solve, PV and
// the two dS sweeps; the shifted dual updates and the vector-cotangent sweeps
// run in tc_rowsum.cuh.
// Epilogue warps: 16 for PV (one CTA per SM, each warp 32 columns of a chunk),
// 8 for the others (each warp 64 columns; the online LSE sweep runs two CTAs per
// SM, the dS modes need the registers); then the loader and the MMA issuers.
__host__ __device__ constexpr int nepi(int m) { return m == simt::PV ? 16 : 8; }
constexpr int TILE = 16384;  // one 128 x 64 bf16 tile
constexpr long long kWaitBudget = 4000000000LL;  // clock cycles (about 2 s)

struct Maps {
    CUtensorMap A, B, A2, B2, X, AR, AC;  // AR, AC: the modifier's K16 operands (DS1)
};

__host__ __device__ constexpr bool is_ds(int m) { return m == DS1 || m == DSD; }
__host__ __device__ constexpr bool has_x(int m) { return m == PV || is_ds(m); }
// the epilogue warps, the loader, the score-MMA issuer, and for the modes with
// a P X contraction a second issuer for it
__host__ __device__ constexpr int nthreads(int m) { return (nepi(m) + (has_x(m) ? 3 : 2)) * 32; }
// operand stages: five for PV and DS1 (their P tiles live in TMEM, which leaves
// the shared memory to the stages), four for the others
constexpr int NST_MAX = 5;
__host__ __device__ constexpr int nst(int m) { return (m == PV || m == DS1) ? 5 : 4; }
__host__ __device__ constexpr int nsb(int m) { return is_ds(m) ? 1 : 2; }
// DS1 with at most five modifier terms adds the modifier to G on the tensor
// core: one more K16 step of the dO V^T contraction whose operands, prepared
// once per sweep in global memory and brought in by TMA with the other
// operands, hold per row (rv_hi, rv_hi, rv_lo) and per column (cv_hi, cv_lo,
// cv_hi) of every term (bf16 halves, rv = rv_hi + rv_lo), so that
//   sum_k rv_k cv_k ~ sum_k rv_hi cv_hi + rv_hi cv_lo + rv_lo cv_hi
// to about 2^-16 of each product, far below the bf16 rounding of dS.
__host__ __device__ constexpr bool aug(int m, int nt) { return m == DS1 && nt > 0 && 3 * nt <= 16; }
// PV adds the column dual to its scores the same way, in one more K16 step of
// the score contraction: a constant row-block operand [1, 1, 1, 0, ...] against
// the chunk's operand rows, which hold a three-way bf16 split of dual / c (c the
// score scale; -1e30 on masked tokens), so its epilogue reads no column vector.
__host__ __device__ constexpr bool augs(int m) { return m == PV; }
__host__ __device__ constexpr bool has_aug(int m, int nt) { return aug(m, nt) || augs(m); }
// column vectors staged per operand stage
__host__ __device__ constexpr int ncv(int m, int nt) {
    return m == DS1 ? (aug(m, nt) ? 1 : 1 + nt) : (m == DSD ? 2 * MAXT : 1);
}
__host__ __device__ constexpr int stage_bytes(int m) {
    return TILE * (1 + (is_ds(m) ? 1 : 0) + (m == PV ? 1 : 0));
}
__host__ __device__ constexpr int tmem_cols(int m) { return has_x(m) ? 512 : 256; }

// row-block operand buffers: two (tile parity) of A for the modes without a second
// score operand; one of A and A2 for the dS modes (their shared memory is full)
__host__ __device__ constexpr int nab(int m) { return is_ds(m) ? 1 : 2; }
// CTAs per SM (the online LSE sweep fits twice)
__host__ __device__ constexpr int ctas_per_sm(int m) { return m == LSE ? 2 : 1; }

// shared-memory carve-up (offsets from a 1024-aligned base)
__host__ __device__ constexpr int off_a(int m, int i) { return TILE * i; }
__host__ __device__ constexpr int off_a2(int m) { return TILE; }
__host__ __device__ constexpr int off_stage(int m) { return 2 * TILE; }
__host__ __device__ constexpr int off_cv(int m) { return off_stage(m) + nst(m) * stage_bytes(m); }
// the modifier's K16 operand tiles (aug): the row block's, then one per operand
// stage, 4 KB each (128 rows x 32 bytes), 1024-aligned
constexpr int AUG_BYTES = 4096;
__host__ __device__ constexpr int off_aug(int m, int nt) {
    return (off_cv(m) + nst(m) * ncv(m, nt) * 128 * 4 + 1023) / 1024 * 1024;
}
__host__ __device__ constexpr int off_red(int m, int nt) {
    return has_aug(m, nt) ? off_aug(m, nt) + (1 + nst(m)) * AUG_BYTES : off_cv(m) + nst(m) * ncv(m, nt) * 128 * 4;
}
__host__ __device__ constexpr int off_bar(int m, int nt) { return off_red(m, nt) + 2 * 4 * 128 * 4; }
__host__ __device__ constexpr int smem_bytes(int m, int nt) { return off_bar(m, nt) + 64 * 8 + 64 + 1024; }

// barrier slots (pairs indexed by tile parity, chunk parity or buffer)
enum { B_AFULL = 0, B_AEMPTY = 2, B_FULL = 4, B_EMPTY = B_FULL + NST_MAX, B_SFULL = B_EMPTY + NST_MAX,
       B_SEMPTY = B_SFULL + 2, B_PFULL = B_SEMPTY + 2, B_PEMPTY = B_PFULL + 2, B_OFULL = B_PEMPTY + 2,
       B_OEMPTY = B_OFULL + 2, B_DRAIN = B_OEMPTY + 2, B_EPI = B_DRAIN + 1, NBAR = B_EPI + 1 };
static_assert(NBAR <= 64, "barrier area");

struct Ctl {
    uint64_t* bar;
    volatile int* abort;
    int* status;
    __device__ bool wait(int slot, uint32_t parity) {
        if (*abort) return false;
        if (tc::mbar_wait(bar + slot, parity, kWaitBudget)) return true;
        *abort = 1;
        if (status) atomicCAS(status, 0, (int)SA_ERR_TIMEOUT);
        return false;
    }
    // every epilogue warp arrives once (after its lanes converge), then all
    // lanes wait (bounded) for the phase
    __device__ bool epi_sync(uint32_t& phase) {
        __syncwarp();
        if ((threadIdx.x & 31) == 0) tc::mbar_arrive(bar + B_EPI);
        const bool ok = wait(B_EPI, phase & 1);
        ++phase;
        return ok;
    }
};

// the chunk's column vector k (128 floats) in stage s
__device__ __forceinline__ float* colvec(uint8_t* sm, int mode, int nt, int s, int k) {
    return reinterpret_cast<float*>(sm + off_cv(mode)) + (s * ncv(mode, nt) + k) * 128;
}

// Exponent arguments (log2 units) of one thread's 32 columns:
// x_j = c2 * s_j + (ce_j + rd2), -inf off the band or past L when `partial`.
__device__ __forceinline__ void group_args(const float (&sv)[32], const float* ce, float rd2,
                                           float c2, bool partial, int r, int cg, int W, int L,
                                           float (&x)[32]) {
    const uint64_t c2p = tc::pk2(c2, c2), rdp = tc::pk2(rd2, rd2);
    const float4* c4 = reinterpret_cast<const float4*>(ce);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 cv = c4[q];
        const uint64_t b0 = tc::add2(tc::pk2(cv.x, cv.y), rdp);
        const uint64_t b1 = tc::add2(tc::pk2(cv.z, cv.w), rdp);
        tc::upk2(tc::fma2(tc::pk2(sv[4 * q], sv[4 * q + 1]), c2p, b0), x[4 * q], x[4 * q + 1]);
        tc::upk2(tc::fma2(tc::pk2(sv[4 * q + 2], sv[4 * q + 3]), c2p, b1), x[4 * q + 2],
                 x[4 * q + 3]);
    }
    if (partial) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int d = r - (cg + j);
            if ((unsigned)(d + W) > (unsigned)(2 * W) || cg + j >= L) x[j] = -INFINITY;
        }
    }
}

// The same with the column dual already in the score (s_j' = s_j + ce_j / c2):
// x_j = c2 * s_j' + rd2.
__device__ __forceinline__ void group_args_s(const float (&sv)[32], float rd2, float c2, bool partial,
                                             int r, int cg, int W, int L, float (&x)[32]) {
    const uint64_t c2p = tc::pk2(c2, c2), rdp = tc::pk2(rd2, rd2);
#pragma unroll
    for (int q = 0; q < 16; ++q)
        tc::upk2(tc::fma2(tc::pk2(sv[2 * q], sv[2 * q + 1]), c2p, rdp), x[2 * q], x[2 * q + 1]);
    if (partial) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int d = r - (cg + j);
            if ((unsigned)(d + W) > (unsigned)(2 * W) || cg + j >= L) x[j] = -INFINITY;
        }
    }
}

// ---------------------------------------------------------------------------
// NT: number of modifier (DS1) or staircase (DSD) terms, 2R; 0 for the other modes.
// Persistent: each CTA walks a contiguous range of (problem, row block) tiles;
// the chunk pipelines (operand stages, score buffers, P buffers) run on one chunk
// counter across tiles, the row-block operand is double-buffered by tile parity
// (single for the dS modes), and the output accumulator of the PV-shaped modes
// is double-buffered in TMEM, so one tile's setup overlaps the previous tile.
template <int MODE, bool ONLINE, int NT>
__global__ void __launch_bounds__(nthreads(MODE), ctas_per_sm(MODE)) tc_band_sweep(const SweepArgs a,
                                                         const __grid_constant__ Maps maps,
                                                         int* status, int BH) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    constexpr int NST = nst(MODE), NSB = nsb(MODE), NAB = nab(MODE);
    constexpr bool DS = is_ds(MODE), HASX = has_x(MODE);
    constexpr int NEPI = nepi(MODE), NPART = NEPI / 4, PW = 128 / NPART, NG = PW / 32;
    constexpr int W_LOAD = NEPI, W_MMA = NEPI + 1, W_MMA2 = NEPI + 2;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + off_bar(MODE, NT));
    uint32_t* tbase = reinterpret_cast<uint32_t*>(sm + off_bar(MODE, NT) + 64 * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tbase + 1);
    float* red = reinterpret_cast<float*>(sm + off_red(MODE, NT));
    static_assert((MODE == LSE && ONLINE) || MODE == PV || MODE == DS1 || MODE == DSD,
                  "the shifted dual updates and WSUM run in tc_rowsum.cuh");
    constexpr bool AUG = aug(MODE, NT), AUGS = augs(MODE), HAUG = has_aug(MODE, NT);
    static_assert(smem_bytes(MODE, NT) <= 227 * 1024 && smem_bytes(MODE, NT) * ctas_per_sm(MODE) <= 228 * 1024,
                  "shared memory");
    static_assert(NST <= NST_MAX, "stage barriers");
    // the column dual is the chunk's only column vector
    constexpr bool CPA = MODE == LSE || (MODE == DS1 && AUG);
    Ctl ctl{bar, abort_flag, status};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = a.L, W = a.W;
    const int nblk = (L + 127) / 128;
    // this CTA's contiguous tile range [t0, t1)
    const int ntiles = BH * nblk;
    const int t0 = (int)(((long long)blockIdx.x * ntiles) / gridDim.x);
    const int t1 = (int)(((long long)(blockIdx.x + 1) * ntiles) / gridDim.x);
    const int ntl = t1 - t0;
    // geometry of a tile; the tiles of the range are walked with a (batch, head,
    // row block) cursor, so that no role divides by a runtime value per tile
    struct Tile {
        int bh, r0, cbeg, cend, nch;
        const uint8_t* mk;
    };
    struct Cursor {
        int rb, h, b;
        __device__ void next(int nb, int H) {
            if (++rb == nb) {
                rb = 0;
                if (++h == H) { h = 0; ++b; }
            }
        }
    };
    const Cursor cur0{t0 % nblk, (t0 / nblk) % a.H, (t0 / nblk) / a.H};
    auto tile = [&](const Cursor& c) {
        Tile g;
        g.bh = c.b * a.H + c.h;
        g.r0 = c.rb * 128;
        g.cbeg = max(0, g.r0 - W);
        g.cend = min(L, g.r0 + 127 + W + 1);
        g.nch = (g.cend - g.cbeg + 127) / 128;
        g.mk = a.mask ? a.mask + (size_t)c.b * L : nullptr;
        return g;
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bar + B_AFULL + i, 1);
            tc::mbar_init(bar + B_AEMPTY + i, 1);
            tc::mbar_init(bar + B_SFULL + i, 1);
            tc::mbar_init(bar + B_SEMPTY + i, NEPI);
            tc::mbar_init(bar + B_PFULL + i, NEPI);
            tc::mbar_init(bar + B_PEMPTY + i, 1);
            tc::mbar_init(bar + B_OFULL + i, 1);
            tc::mbar_init(bar + B_OEMPTY + i, NEPI);
        }
        for (int s = 0; s < NST; ++s) {
            tc::mbar_init(bar + B_FULL + s, AUGS ? 1 : 33);  // the TMA bytes (+ 32 lanes' vectors)
            tc::mbar_init(bar + B_EMPTY + s, NEPI + 1);
        }
        tc::mbar_init(bar + B_DRAIN, HASX ? 2 : 1);  // every MMA issuer
        tc::mbar_init(bar + B_EPI, NEPI);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tbase, tmem_cols(MODE));
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tm = *tbase;
    // TMEM columns: S buffer b at 128*b (DS: S at 0, G at 128); O buffer ob at
    // 256 + 64*ob; P (or dS) buffer pb, 128 bf16 per row, at 384 + 64*pb
    const uint32_t tS = tm, tG = tm + 128, tO = tm + 256, tP = tm + 384;
    // The set-up above overlaps the previous kernel's tail; every global
    // access comes after this wait.  Then the next kernel may begin launching.
    tc::grid_dep_wait();
    tc::grid_dep_launch();

    if (warp == W_LOAD) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            tc::prefetch_tmap(&maps.A);
            tc::prefetch_tmap(&maps.B);
        }
        int gc = 0, issued = 0, a_issued = 0;
        bool ok = true;
        Cursor cur = cur0;
        for (int it = 0; ok && it < ntl; ++it, cur.next(nblk, a.H)) {
            const Tile tl = tile(cur);
            const int ab = it % NAB;
            if (lane == 0) {
                if (it >= NAB && !ctl.wait(B_AEMPTY + ab, ((it / NAB) - 1) & 1)) ok = false;
                if (ok) {
                    // the row-block operand rows: per tile (DS1), or the constant one
                    // once, with the first tile (PV)
                    const bool ld_ar = AUG || (AUGS && it == 0);
                    tc::mbar_expect_tx(bar + B_AFULL + ab, TILE * (DS ? 2 : 1) + (ld_ar ? AUG_BYTES : 0));
                    tc::tma_load_3d(sm + off_a(MODE, ab), &maps.A, bar + B_AFULL + ab, 0, tl.r0, tl.bh);
                    if (DS) tc::tma_load_3d(sm + off_a2(MODE), &maps.A2, bar + B_AFULL + ab, 0, tl.r0, tl.bh);
                    if (AUG) tc::tma_load_3d(sm + off_aug(MODE, NT), &maps.AR, bar + B_AFULL + ab, 0, tl.r0, tl.bh);
                    if (AUGS && it == 0) tc::tma_load_3d(sm + off_aug(MODE, NT), &maps.AR, bar + B_AFULL + ab, 0, 0, 0);
                    a_issued = it + 1;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            for (int c = 0; ok && c < tl.nch; ++c, ++gc) {
                const int s = gc % NST;
                if (gc >= NST && !ctl.wait(B_EMPTY + s, ((gc / NST) - 1) & 1)) { ok = false; break; }
                issued = gc + 1;
                const int c0 = tl.cbeg + 128 * c, cend = tl.cend, bh = tl.bh;
                const uint8_t* mk = tl.mk;
                uint8_t* st = sm + off_stage(MODE) + s * stage_bytes(MODE);
                if (lane == 0) {
                    tc::mbar_expect_tx(bar + B_FULL + s, stage_bytes(MODE) + (HAUG ? AUG_BYTES : 0));
                    tc::tma_load_3d(st, &maps.B, bar + B_FULL + s, 0, c0, bh);
                    if (DS) tc::tma_load_3d(st + TILE, &maps.B2, bar + B_FULL + s, 0, c0, bh);
                    if (HAUG)
                        tc::tma_load_3d(sm + off_aug(MODE, NT) + AUG_BYTES * (1 + s), &maps.AC,
                                        bar + B_FULL + s, 0, c0, bh);
                    if (MODE == PV) tc::tma_load_3d(st + TILE, &maps.X, bar + B_FULL + s, 0, c0, bh);
                }
                if (AUGS) continue;  // no column vector
                // Column vectors.  The modes whose only one is the column dual copy it
                // from its working copy (log2(e) times the dual, -inf on masked
                // tokens) by 4-byte cp.async, counted on the stage's mbarrier, so the
                // loader never waits for a global load; columns past L are
                // zero-filled and excluded by the epilogue's band test.
                if (CPA && a.cdw.p) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int col = c0 + 32 * k + lane;
                        const bool in = col < L;
                        tc::cp_async4(colvec(sm, MODE, NT, s, 0) + 32 * k + lane,
                                      a.cdw.p + (long long)bh * a.cdw.s + (in ? col : 0), in);
                    }
                    tc::cp_async_arrive(bar + B_FULL + s);
                    continue;
                }
                // Otherwise: -inf / 0 outside [cbeg, cend) and on masked columns.
                // Every load of the chunk (4 columns per lane, each vector, the mask)
                // is issued before any value is used or stored.
                {
                    constexpr int NV = MODE == DS1 ? 1 + NT : (MODE == DSD ? 2 * NT : 1);
                    float val[4][NV > 0 ? NV : 1];
                    bool inr[4], mok[4];
    #pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int col = c0 + 32 * k + lane;
                        inr[k] = col < cend;
                        mok[k] = true;
    #pragma unroll
                        for (int e = 0; e < NV; ++e) val[k][e] = 0.f;
                        if (inr[k]) {
                            if (mk) mok[k] = mk[col] != 0;
                            if (MODE != DSD) val[k][0] = a.cd.at(bh, col);
                            if (MODE == DS1 && !AUG) {
    #pragma unroll
                                for (int e = 0; e < NT; ++e) val[k][1 + e] = a.cv[e].p ? a.cv[e].at(bh, col) : 1.f;
                            }
                            if (MODE == DSD) {
    #pragma unroll
                                for (int e = 0; e < NT; ++e) {
                                    val[k][e] = a.ec[e].at(bh, col);
                                    val[k][NT + e] = a.cc[e].p ? a.cc[e].at(bh, col) : 0.f;
                                }
                            }
                        }
                    }
    #pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int t = 32 * k + lane;
                        const bool ok = inr[k] && mok[k];
                        colvec(sm, MODE, NT, s, 0)[t] =
                            (MODE == DSD) ? 0.f : (ok ? val[k][0] * kLog2e : -INFINITY);
                        if (MODE == DS1 && !AUG) {
    #pragma unroll
                            for (int e = 0; e < NT; ++e) colvec(sm, MODE, NT, s, 1 + e)[t] = ok ? val[k][1 + e] : 0.f;
                        }
                        if (MODE == DSD) {
    #pragma unroll
                            for (int e = 0; e < NT; ++e) {
                                colvec(sm, MODE, NT, s, e)[t] = ok ? val[k][e] * kLog2e : -INFINITY;
                                colvec(sm, MODE, NT, s, MAXT + e)[t] = ok ? val[k][NT + e] : 0.f;
                            }
                        }
                    }
                }
                tc::mbar_arrive(bar + B_FULL + s);
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");  // nothing in flight at exit
        // after an abort, let the tile loads already issued land before teardown
        if (lane == 0 && *abort_flag) {
            for (int x = max(0, a_issued - NAB); x < a_issued; ++x)
                tc::mbar_wait(bar + B_AFULL + x % NAB, (x / NAB) & 1, kWaitBudget);
            for (int x = max(0, issued - NST); x < issued; ++x)
                tc::mbar_wait(bar + B_FULL + x % NST, (x / NST) & 1, kWaitBudget);
        }
        __syncwarp();
    } else if (warp == W_MMA || (HASX && warp == W_MMA2)) {
        // ------------------------------------------------------------ MMA issuers
        // The whole warp runs the loop (uniform control flow and values); one
        // elected lane issues the MMAs and commits.  W_MMA issues the score
        // contractions; for the modes with one, W_MMA2 issues P X, so that
        // neither stream of MMA instructions waits behind the other's issue.
        const bool pvw = HASX && warp == W_MMA2;
        {
            const uint32_t id_s = tc::idesc_bf16(128, 128, false, false);
            const uint32_t id_o = tc::idesc_bf16(128, 64, false, true);
            // descriptors built once; offsets are added in 16-byte units
            const uint64_t dA0 = tc::sdesc_sw128(tc::smem_u32(sm), 16, 1024);
            const uint64_t dA2 = tc::sdesc_sw128(tc::smem_u32(sm + off_a2(MODE)), 16, 1024);
            const uint64_t dStK = tc::sdesc_sw128(tc::smem_u32(sm + off_stage(MODE)), 16, 1024);
            const uint64_t dStMN = tc::sdesc_sw128(tc::smem_u32(sm + off_stage(MODE)), TILE, 1024);
            const uint64_t dAug = tc::sdesc_sw32(tc::smem_u32(sm + off_aug(MODE, NT)));
            // O += P X of chunk c (global chunk g) of tile it (nch chunks)
            auto issue_pv = [&](int g, int it, int c, int nch) -> bool {
                const int pb = g & 1, s = g % NST, ob = it & 1;
                // the epilogue has read this O buffer's previous tile (it - 2)
                if (c == 0 && it >= 2 && !ctl.wait(B_OEMPTY + ob, ((it >> 1) - 1) & 1)) return false;
                if (!ctl.wait(B_PFULL + pb, (g >> 1) & 1)) return false;
                tc::tc_fence_after();
                const uint64_t dX = tc::sdesc_add(dStMN, s * stage_bytes(MODE) + (MODE == PV ? TILE : 0));
                if (tc::elect_one()) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {  // A = P from TMEM, 16 chunk columns per step
                        tc::mma_bf16_ts(tO + 64 * ob, tP + 64 * pb + 8 * k, tc::sdesc_add(dX, k * 2048), id_o,
                                        (c > 0 || k > 0) ? 1u : 0u);
                    }
                    tc::tc_commit(bar + B_PEMPTY + pb);
                    tc::tc_commit(bar + B_EMPTY + s);
                    if (c == nch - 1) tc::tc_commit(bar + B_OFULL + ob);
                }
                __syncwarp();
                return true;
            };
            bool ok = true;
            int gc = 0;
            Cursor cur = cur0;
            if (pvw) {
                for (int it = 0; ok && it < ntl; ++it, cur.next(nblk, a.H)) {
                    const Tile tl = tile(cur);
                    for (int c = 0; c < tl.nch; ++c, ++gc) {
                        // the stage's X tile has landed (its phase cannot move on before
                        // this warp's commit releases the stage)
                        if (!ctl.wait(B_FULL + gc % NST, (gc / NST) & 1)) { ok = false; break; }
                        if (!issue_pv(gc, it, c, tl.nch)) { ok = false; break; }
                    }
                }
            } else {
                for (int it = 0; ok && it < ntl; ++it, cur.next(nblk, a.H)) {
                    const Tile tl = tile(cur);
                    const int ab = it % NAB;
                    if (!ctl.wait(B_AFULL + ab, (it / NAB) & 1)) { ok = false; break; }
                    const uint64_t dA = tc::sdesc_add(dA0, off_a(MODE, ab));
                    for (int c = 0; c < tl.nch; ++c, ++gc) {
                        const int s = gc % NST, b = gc % NSB;
                        if (!ctl.wait(B_FULL + s, (gc / NST) & 1)) { ok = false; break; }
                        if (gc >= NSB && !ctl.wait(B_SEMPTY + b, ((gc / NSB) - 1) & 1)) { ok = false; break; }
                        tc::tc_fence_after();
                        const uint64_t dB = tc::sdesc_add(dStK, s * stage_bytes(MODE));
                        if (tc::elect_one()) {
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                tc::mma_bf16(tS + 128 * b, tc::sdesc_add(dA, 32 * k), tc::sdesc_add(dB, 32 * k),
                                             id_s, k > 0);
                            if (AUGS)  // + the column duals
                                tc::mma_bf16(tS + 128 * b, dAug, tc::sdesc_add(dAug, AUG_BYTES * (1 + s)), id_s, 1u);
                            if (DS) {
#pragma unroll
                                for (int k = 0; k < 4; ++k)
                                    tc::mma_bf16(tG, tc::sdesc_add(dA2, 32 * k), tc::sdesc_add(dB, TILE + 32 * k),
                                                 id_s, k > 0);
                                if (AUG)  // + the modifier, one more K16 step
                                    tc::mma_bf16(tG, dAug, tc::sdesc_add(dAug, AUG_BYTES * (1 + s)), id_s, 1u);
                            }
                            tc::tc_commit(bar + B_SFULL + b);
                            if (!HASX) tc::tc_commit(bar + B_EMPTY + s);
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                    if (tc::elect_one()) tc::tc_commit(bar + B_AEMPTY + ab);  // every score MMA of the tile has read A
                    __syncwarp();
                }
            }
            // drain: every MMA issued above has completed once this arrives
            if (tc::elect_one()) tc::tc_commit(bar + B_DRAIN);
            __syncwarp();
            tc::mbar_wait(bar + B_DRAIN, 0, kWaitBudget);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int qd = warp & 3, pt = warp >> 2;  // part pt: columns PW*pt..PW*pt+PW-1 of a chunk
        const int lr = qd * 32 + lane;            // local row
        const uint32_t lanebase = (uint32_t)(qd * 32) << 16;
        const float c2 = a.c2;
        constexpr int OWY = 64 / NPART;
        int gc = 0;
        uint32_t eph = 0;
        bool ok = true;
        // Row-side values of the tile in progress; the next tile's are loaded as
        // soon as the chunk loop of the current one no longer needs them.
        float rd2 = 0.f;
        bool rok = false;
        float rmod[NT > 0 ? NT : 1], rmod2[NT > 0 ? NT : 1];
        auto load_rows = [&](const Tile& tl) {
            const int r = tl.r0 + lr;
            rok = r < L && (tl.mk == nullptr || tl.mk[r] != 0);
            rd2 = 0.f;
            if (r < L) {
                if (MODE != LSE && MODE != DSD) rd2 = a.rd.at(tl.bh, r) * kLog2e;
            }
#pragma unroll
            for (int k = 0; k < NT; ++k) {
                rmod[k] = 0.f;
                rmod2[k] = 0.f;
                if (r < L) {
                    if (MODE == DS1 && !AUG) rmod[k] = a.rv[k].p ? a.rv[k].at(tl.bh, r) : 1.f;
                    if (MODE == DSD) {
                        rmod[k] = a.er[k].at(tl.bh, r) * kLog2e;
                        rmod2[k] = a.cr[k].p ? a.cr[k].at(tl.bh, r) : 0.f;
                    }
                }
            }
        };
        if (ntl >= 1) load_rows(tile(cur0));
        // dS modes: a tile's dQ / dK rows are read out of TMEM after the next
        // tile's first chunk (or after the last tile), by when the tile's last
        // dS X MMA has long completed; O is double-buffered, and the MMA needs
        // buffer it & 1 again only for tile it + 2
        bool pend = false;
        int p_it = 0, p_bh = 0, p_r = 0;
        bool p_rok = false;
        auto ds_finish = [&](int fit, int fbh, int fr, bool frok) -> bool {
            constexpr int OW = 64 / NPART;
            const int ob = fit & 1;
            if (!ctl.wait(B_OFULL + ob, (fit >> 1) & 1)) return false;
            float o[OW];
            {
                tc::tc_fence_after();
                uint32_t u0[OW];
                if constexpr (OW == 32) tc::tmem_ld32(tO + 64 * ob + lanebase + OW * pt, u0);
                else tc::tmem_ld16(tO + 64 * ob + lanebase + OW * pt, u0);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < OW; ++j) o[j] = __uint_as_float(u0[j]);
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar + B_OEMPTY + ob);
            }
#pragma unroll
            for (int j = 0; j < OW; ++j) o[j] = frok ? o[j] * a.out_scale : 0.f;
            float* accr = (a.acc && fr < L) ? a.acc + ((size_t)fbh * L + fr) * 64 + OW * pt : nullptr;
            if (accr && a.acc_in) {
#pragma unroll
                for (int q = 0; q < OW / 4; ++q) {
                    const float4 p = reinterpret_cast<const float4*>(accr)[q];
                    o[4 * q] += p.x; o[4 * q + 1] += p.y; o[4 * q + 2] += p.z; o[4 * q + 3] += p.w;
                }
            }
            if (accr && a.acc_out) {
#pragma unroll
                for (int q = 0; q < OW / 4; ++q)
                    reinterpret_cast<float4*>(accr)[q] =
                        make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
            } else if (fr < L && SA_BOUNDS(fbh < BH && fr >= 0, status)) {
                __nv_bfloat16* outp =
                    reinterpret_cast<__nv_bfloat16*>(a.out_mat) + ((size_t)fbh * L + fr) * 64 + OW * pt;
#pragma unroll
                for (int q = 0; q < OW / 8; ++q) {
                    uint4 w;
                    w.x = tc::pack_bf16(o[8 * q + 0], o[8 * q + 1]);
                    w.y = tc::pack_bf16(o[8 * q + 2], o[8 * q + 3]);
                    w.z = tc::pack_bf16(o[8 * q + 4], o[8 * q + 5]);
                    w.w = tc::pack_bf16(o[8 * q + 6], o[8 * q + 7]);
                    reinterpret_cast<uint4*>(outp)[q] = w;
                }
            }
            return true;
        };
        Cursor cur = cur0;
        for (int it = 0; ok && it < ntl; ++it, cur.next(nblk, a.H)) {
            const Tile tl = tile(cur);
            const int bh = tl.bh, r0 = tl.r0, cbeg = tl.cbeg, nch = tl.nch;
            const int r = r0 + lr;              // global row
            const int rw0 = r0 + qd * 32;       // first row of this warp
            float m = -INFINITY, acc = 0.f;   // LSE online max / running sum

            for (int c = 0; c < nch; ++c, ++gc) {
                const int s = gc % NST, b = gc % NSB, pb = gc & 1;
                if (!ctl.wait(B_FULL + s, (gc / NST) & 1)) { ok = false; break; }
                if (!ctl.wait(B_SFULL + b, (gc / NSB) & 1)) { ok = false; break; }
                if (HASX && gc >= 2 && !ctl.wait(B_PEMPTY + pb, ((gc >> 1) - 1) & 1)) { ok = false; break; }
                tc::tc_fence_after();
                const int c0 = cbeg + 128 * c;
                const float* cvs = colvec(sm, MODE, NT, s, 0) + PW * pt;
                // Modes with a matrix output (one CTA per SM, registers to spare) read all
                // of this warp's scores of the chunk (and the dO V^T tile) with one wait
                // and free the TMEM buffer at once; the others read a group at a time.
                constexpr bool UPFRONT = MODE == PV;
                uint32_t su[UPFRONT ? NG : 1][32], gu[UPFRONT && DS ? NG : 1][32];
                if (UPFRONT) {
    #pragma unroll
                    for (int g = 0; g < NG; ++g) {
                        tc::tmem_ld32(tS + 128 * b + lanebase + PW * pt + 32 * g, su[UPFRONT ? g : 0]);
                        if (DS) tc::tmem_ld32(tG + lanebase + PW * pt + 32 * g, gu[UPFRONT && DS ? g : 0]);
                    }
                    tc::tmem_wait_ld();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar + B_SEMPTY + b);
                }
    #pragma unroll 1
                for (int g = 0; g < NG; ++g) {
                    float sv[32], gv[DS ? 32 : 1], pv[32];
                    if (UPFRONT) {
                        // select, not index: the loop over g stays rolled and su in registers
    #pragma unroll
                        for (int j = 0; j < 32; ++j)
                            sv[j] = __uint_as_float(g ? su[(UPFRONT && NG > 1) ? 1 : 0][j] : su[0][j]);
                    } else {
                        if (SA_BOUNDS(128 * b + PW * pt + 32 * g + 32 <= tmem_cols(MODE), status))
                            tc::tmem_ld32(tS + 128 * b + lanebase + PW * pt + 32 * g, su[0]);
                        if (DS) tc::tmem_ld32(tG + lanebase + PW * pt + 32 * g, gu[0]);
                        tc::tmem_wait_ld();
    #pragma unroll
                        for (int j = 0; j < 32; ++j) sv[j] = __uint_as_float(su[0][j]);
                        if (DS) {
    #pragma unroll
                            for (int j = 0; j < 32; ++j)
                                gv[j] = (MODE == DS1 && a.g_off) ? 0.f : __uint_as_float(gu[0][j]);
                        }
                        if (g == NG - 1) {  // every TMEM read of this chunk is done
                            tc::tc_fence_before();
                            __syncwarp();
                            if (lane == 0) tc::mbar_arrive(bar + B_SEMPTY + b);
                        }
                    }
                    // band test for this warp's 32 rows x these 32 columns (warp-uniform)
                    const int cg = c0 + PW * pt + 32 * g;
                    const bool all_in = (cg >= rw0 + 31 - W) && (cg + 31 <= rw0 + W) && cg + 31 < L;
                    const bool all_out = (cg + 31 < rw0 - W) || (cg > rw0 + 31 + W) || cg >= L;
                    const float* ce = cvs + 32 * g;
                    if (MODE == LSE || MODE == PV) {
                        if (all_out) {
                            if (MODE == PV) {
    #pragma unroll
                                for (int j = 0; j < 32; ++j) pv[j] = 0.f;
                            }
                        } else {
                            float x[32];
                            if (AUGS) group_args_s(sv, rd2, c2, !all_in, r, cg, W, L, x);
                            else group_args(sv, ce, rd2, c2, !all_in, r, cg, W, L, x);
                            if (MODE == LSE) {
                                float mloc = -INFINITY;
    #pragma unroll
                                for (int j = 0; j < 32; ++j) mloc = fmaxf(mloc, x[j]);
                                if (mloc > m) {
                                    acc *= ex2(m - mloc);
                                    m = mloc;
                                }
                                if (m != -INFINITY) {
    #pragma unroll
                                    for (int j = 0; j < 32; ++j) acc += ex2(x[j] - m);
                                }
                            } else {  // PV
    #pragma unroll
                                for (int j = 0; j < 32; ++j) pv[j] = ex2(x[j]);
                            }
                        }
                    } else if (all_out) {
    #pragma unroll
                        for (int j = 0; j < 32; ++j) pv[j] = 0.f;
                    } else if (MODE == DS1 && AUG) {
                        // dS = P * M, M = G + sum_k rv_k[row] cv_k[col] from the contraction
                        float x[32];
                        group_args(sv, ce, rd2, c2, !all_in, r, cg, W, L, x);
    #pragma unroll
                        for (int j = 0; j < 32; ++j) pv[j] = ex2(x[j]) * gv[j];
                    } else if (MODE == DS1) {
                        // dS = P * M,  M = G + sum_k rv_k[row] cv_k[col]
                        float x[32];
                        group_args(sv, ce, rd2, c2, !all_in, r, cg, W, L, x);
    #pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            uint64_t m01 = tc::pk2(gv[4 * q], gv[4 * q + 1]);
                            uint64_t m23 = tc::pk2(gv[4 * q + 2], gv[4 * q + 3]);
    #pragma unroll
                            for (int k = 0; k < NT; ++k) {
                                const float4 cv = reinterpret_cast<const float4*>(
                                    colvec(sm, MODE, NT, s, 1 + k) + PW * pt + 32 * g)[q];
                                const uint64_t rk = tc::pk2(rmod[k], rmod[k]);
                                m01 = tc::fma2(rk, tc::pk2(cv.x, cv.y), m01);
                                m23 = tc::fma2(rk, tc::pk2(cv.z, cv.w), m23);
                            }
                            float M0, M1, M2, M3;
                            tc::upk2(m01, M0, M1);
                            tc::upk2(m23, M2, M3);
                            pv[4 * q] = ex2(x[4 * q]) * M0;
                            pv[4 * q + 1] = ex2(x[4 * q + 1]) * M1;
                            pv[4 * q + 2] = ex2(x[4 * q + 2]) * M2;
                            pv[4 * q + 3] = ex2(x[4 * q + 3]) * M3;
                        }
                    } else {
                        // DSD: dS = sum_k exp(S + er_k[row] + ec_k[col]) (g_k G + cr_k[row] + cc_k[col])
                        const uint64_t c2p = tc::pk2(c2, c2);
    #pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float v4[4] = {0.f, 0.f, 0.f, 0.f};
    #pragma unroll
                            for (int k = 0; k < NT; ++k) {
                                const float4 ev = reinterpret_cast<const float4*>(
                                    colvec(sm, MODE, NT, s, k) + PW * pt + 32 * g)[q];
                                const float4 cv = reinterpret_cast<const float4*>(
                                    colvec(sm, MODE, NT, s, MAXT + k) + PW * pt + 32 * g)[q];
                                const uint64_t rk = tc::pk2(rmod[k], rmod[k]);
                                float x0, x1, x2, x3;
                                tc::upk2(tc::fma2(tc::pk2(sv[4 * q], sv[4 * q + 1]), c2p,
                                                  tc::add2(tc::pk2(ev.x, ev.y), rk)), x0, x1);
                                tc::upk2(tc::fma2(tc::pk2(sv[4 * q + 2], sv[4 * q + 3]), c2p,
                                                  tc::add2(tc::pk2(ev.z, ev.w), rk)), x2, x3);
                                const float gk = a.gk[k], ck = rmod2[k];
                                v4[0] = fmaf(ex2(x0), fmaf(gk, gv[4 * q], ck + cv.x), v4[0]);
                                v4[1] = fmaf(ex2(x1), fmaf(gk, gv[4 * q + 1], ck + cv.y), v4[1]);
                                v4[2] = fmaf(ex2(x2), fmaf(gk, gv[4 * q + 2], ck + cv.z), v4[2]);
                                v4[3] = fmaf(ex2(x3), fmaf(gk, gv[4 * q + 3], ck + cv.w), v4[3]);
                            }
    #pragma unroll
                            for (int e = 0; e < 4; ++e) pv[4 * q + e] = v4[e];
                        }
                        if (!all_in) {
    #pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const int d = r - (cg + j);
                                if ((unsigned)(d + W) > (unsigned)(2 * W)) pv[j] = 0.f;
                            }
                        }
                    }
                    if (HASX) {
                        // the group's 32 columns as 16 bf16 pairs, at TMEM column
                        // (chunk column) / 2 of the P buffer
                        const int jc = PW * pt + 32 * g;  // first column of the group within the chunk
                        uint32_t w[16];
    #pragma unroll
                        for (int q = 0; q < 16; ++q) w[q] = tc::pack_bf16(pv[2 * q], pv[2 * q + 1]);
                        if (SA_BOUNDS(384 + 64 * pb + jc / 2 + 16 <= tmem_cols(MODE), status))
                            tc::tmem_st16(tP + 64 * pb + lanebase + jc / 2, w);
                    }
                }
                if (HASX) {
                    // the stores have landed before the MMA that reads them is issued
                    tc::tmem_wait_st();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar + B_PFULL + pb);
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar + B_EMPTY + s);
                if (DS && c == 0 && pend) {  // the previous tile's rows
                    if (!ds_finish(p_it, p_bh, p_r, p_rok)) { ok = false; break; }
                    pend = false;
                }
            }

            if (!ok) break;
            // what the finish still needs of this tile; then the next tile's rows
            const float rd2f = rd2;
            const bool rokf = rok;
            if (it + 1 < ntl) {
                Cursor nx = cur;
                nx.next(nblk, a.H);
                load_rows(tile(nx));
            }

            // ---------------------------------------------------------- finish
            const float ce_d = a.dustbin ? a.cd.at(bh, L) * kLog2e : 0.f;
            float* rr = red + (it & 1) * 512;  // double-buffered by tile parity
            if (MODE == LSE) {
                // combine the two column halves of each row
                rr[pt * 256 + lr] = m;
                rr[pt * 256 + 128 + lr] = acc;
                if (!ctl.epi_sync(eph)) { ok = false; break; }
                if (pt == 0 && r < L && !*abort_flag) {
                    float m1 = rr[lr], s1 = rr[128 + lr];
                    const float m2 = rr[256 + lr], s2 = rr[384 + lr];
                    lse_merge(m1, s1, m2, s2);
                    if (a.dustbin) lse_merge(m1, s1, a.sd2 + ce_d, 1.f);
                    const float out = -(m1 + lg2(s1)) * kLn2;
                    if (SA_BOUNDS(bh < BH && r >= 0, status)) a.out_vec.at(bh, r) = rokf ? out : 0.f;
                }
            } else if (DS) {
                pend = true;
                p_it = it;
                p_bh = bh;
                p_r = r;
                p_rok = rokf;
            } else {
                // O accumulator of this tile: this warp reads columns OW*pt..OW*pt+OW-1
                // of its lanes, then frees the buffer for tile it + 2
                constexpr int OW = 64 / NPART;
                const int ob = it & 1;
                // PV with a row dot: this thread's slice of the Y row, loaded while
                // the tile's last P X contraction completes
                uint4 yq[MODE == PV ? OWY / 8 : 1];
                if (MODE == PV) {
#pragma unroll
                    for (int q = 0; q < (MODE == PV ? OWY / 8 : 1); ++q) yq[q] = make_uint4(0, 0, 0, 0);
                    if (a.Y && r < L) {
                        const uint4* yp = reinterpret_cast<const uint4*>(
                            reinterpret_cast<const __nv_bfloat16*>(a.Y) + ((size_t)bh * L + r) * 64 + OWY * pt);
#pragma unroll
                        for (int q = 0; q < (MODE == PV ? OWY / 8 : 1); ++q) yq[q] = yp[q];
                    }
                }
                if (!ctl.wait(B_OFULL + ob, (it >> 1) & 1)) { ok = false; break; }
                float o[OW];
                {
                    tc::tc_fence_after();
                    uint32_t u0[OW];
                    if constexpr (OW == 32) tc::tmem_ld32(tO + 64 * ob + lanebase + OW * pt, u0);
                    else tc::tmem_ld16(tO + 64 * ob + lanebase + OW * pt, u0);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < OW; ++j) o[j] = __uint_as_float(u0[j]);
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar + B_OEMPTY + ob);
                }
                const float scale = DS ? a.out_scale : 1.f;
                if (MODE == PV && a.dustbin && a.Xd && rokf) {
                    const float p = ex2(a.sd2 + rd2f + ce_d);
                    const float* xd = a.Xd + (size_t)(bh % a.H) * 64 + OW * pt;
#pragma unroll
                    for (int j = 0; j < OW; ++j) o[j] = fmaf(p, xd[j], o[j]);
                }
#pragma unroll
                for (int j = 0; j < OW; ++j) o[j] = rokf ? o[j] * scale : 0.f;
                float dot = 0.f;
                float* accr = (DS && a.acc && r < L) ? a.acc + ((size_t)bh * L + r) * 64 + OW * pt : nullptr;
                if (DS && accr && a.acc_in) {
#pragma unroll
                    for (int q = 0; q < OW / 4; ++q) {
                        const float4 p = reinterpret_cast<const float4*>(accr)[q];
                        o[4 * q] += p.x; o[4 * q + 1] += p.y; o[4 * q + 2] += p.z; o[4 * q + 3] += p.w;
                    }
                }
                if (DS && accr && a.acc_out) {
#pragma unroll
                    for (int q = 0; q < OW / 4; ++q)
                        reinterpret_cast<float4*>(accr)[q] =
                            make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
                } else if (r < L && SA_BOUNDS(bh < BH && r >= 0, status)) {
                    __nv_bfloat16* outp =
                        reinterpret_cast<__nv_bfloat16*>(a.out_mat) + ((size_t)bh * L + r) * 64 + OW * pt;
#pragma unroll
                    for (int q = 0; q < OW / 8; ++q) {
                        uint4 w;
                        w.x = tc::pack_bf16(o[8 * q + 0], o[8 * q + 1]);
                        w.y = tc::pack_bf16(o[8 * q + 2], o[8 * q + 3]);
                        w.z = tc::pack_bf16(o[8 * q + 4], o[8 * q + 5]);
                        w.w = tc::pack_bf16(o[8 * q + 6], o[8 * q + 7]);
                        reinterpret_cast<uint4*>(outp)[q] = w;
                    }
                    if (MODE == PV && a.Y) {
#pragma unroll
                        for (int q = 0; q < OW / 8; ++q) {
                            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&yq[MODE == PV ? q : 0]);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = __bfloat1622float2(h[e]);
                                dot = fmaf(f.x, o[8 * q + 2 * e], dot);
                                dot = fmaf(f.y, o[8 * q + 2 * e + 1], dot);
                            }
                        }
                    }
                }
                if (MODE == PV && a.Y) {
                    rr[pt * 128 + lr] = dot;
                    if (!ctl.epi_sync(eph)) { ok = false; break; }
                    if (pt == 0 && r < L && a.out_vec.p && !*abort_flag) {
                        float tot = 0.f;
#pragma unroll
                        for (int k = 0; k < NPART; ++k) tot += rr[k * 128 + lr];
                        if (SA_BOUNDS(bh < BH && r >= 0, status)) a.out_vec.at(bh, r) = rokf ? tot : 0.f;
                    }
                }
            }
        }
        if (DS && ok && pend) ds_finish(p_it, p_bh, p_r, p_rok);  // the last tile's rows
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, tmem_cols(MODE));
    }
}

}  // namespace tcs
}  // namespace sa
