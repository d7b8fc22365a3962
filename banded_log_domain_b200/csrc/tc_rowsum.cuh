// Row-sum band sweeps on the tensor cores (bf16 storage): the dual update
// (LSE) and the vector-cotangent sweep (WSUM) of the method, one launch per
// sweep over every (batch, head) problem.
//
//   LSE : out_i = -log sum_j exp(S_ij + cd_j)                   (rd: the shift source)
//   WSUM: out_i = base_i + sgn * mult_i * sum_j exp(S_ij + rd_i + cd_j) w_j
//
// with S = QK^T / (sqrt(d) eps) on the band |i - j| <= W (both tokens valid).
// These are the two sweeps whose per-entry work is one exponential and one
// addition (or FMA) into a row sum.  The exponential rate bounds them from
// below; as measured, the pipeline of loads, MMA issue and barrier hand-offs
// binds first (the same kernel without its epilogue arithmetic takes about
// four fifths of the time).
//
// Layout of the work.  A CTA per SM walks a contiguous range of (problem, row
// block of 128) tiles.  A tile's columns are the chunks r0 - W + 128 c,
// c < nch = ceil((2W + 128) / 128), on one grid for the whole problem, so that
// the next row block of the same problem needs only one new chunk: the K-side
// chunks (TMA tiles with their column-dual operands) sit in a ring of NRING slots and
// a chunk stays until every tile that reads it has (reuse; streaming when W is
// so large that a tile's chunks do not fit the ring).  A slot's EMPTY barrier
// expects 4 arrivals (one per quadrant warp) from each of up to nch uses and
// one MMA commit at the last use; the loader, which knows how many tiles of its
// range will read a chunk, arrives for the uses that will not happen.  Scores go to one
// of four TMEM buffers, one per epilogue part: epilogue warp (quadrant q,
// part p) processes the 32 rows of quadrant q of the chunks assigned to part
// p, from buffer p: a whole 128-column chunk per warp, so the MMA runs up to
// four chunks ahead; the assignment rotates the band-edge chunks over the
// parts.  The four parts' partial row sums of a tile meet in shared memory,
// where a finisher warp adds them and writes the tile's outputs.
//
// Operand traffic.  Q and K tiles come by TMA, and with each K chunk the
// column duals as a 16-wide bf16 operand row per token (a three-way bf16 split
// of dual / c in slots 0-2, c the score scale): a fifth MMA of the chunk, with a
// constant row-block operand [1, 1, 1, 0, ...], adds the column dual to every
// score in TMEM, so the epilogue reads no column vector at all.  The split
// keeps 24 significant bits of the dual; the sum is formed in the fp32
// accumulator.  Masked columns carry -1e30, which drives their terms to 0.
// The per-row data (the rows' working duals, the WSUM base and multiplier)
// and the WSUM weights come by 4-byte cp.async, counted on mbarriers, so the
// loader never waits for a global load.  The duals are read as working copies
// (log2(e) times the dual, -inf on masked tokens, and the operand rows), which
// each LSE sweep writes next to its natural-unit output for the sweep after
// it.  Columns outside [0, L) are zero-filled and excluded by the band-edge
// test.
//
// Exponent shift.  Every term is a plan entry of a plan with unit columns (or
// rows) and so is at most 1 when shifted by the row's previous dual rd_i, so
// each row uses its own shift: the per-entry argument is one FMA,
// c2 * (s + cd_j / c) + rd_i, with all arguments <= 0 up to rounding.
//
// Exponentials: 2^x on the MUFU unit (ex2.approx), and for KP of every 32
// entries of a group that lies inside the band on the FMA pipe: range
// reduction x = n + f, |f| <= 1/2, n by round-to-nearest (adding 1.5 * 2^23),
// 2^f from a degree-5 polynomial fitted by least squares on Chebyshev nodes to
// the relative error (at most 2.2e-7 with fp32 Horner FMAs, the accuracy of
// ex2.approx), and 2^n added to the result's exponent field.  Arguments are
// clamped at -126 (the result is then below 2^-125, nothing next to a row sum
// that holds a term close to 1).
#pragma once

#include "common.cuh"
#include "simt_sweep.cuh"
#include "tc_ptx.cuh"

namespace sa {
namespace tcr {

using simt::SweepArgs;
constexpr int LSE = simt::LSE, WSUM = simt::WSUM;

constexpr int NEPI = 16;                 // epilogue warps: quadrant w % 4, part w / 4
constexpr int W_LOAD = NEPI, W_MMA = NEPI + 1, W_FIN = NEPI + 2;
constexpr int NTHREADS = (NEPI + 3) * 32;
constexpr int NRING = 8;                 // K-chunk ring slots
constexpr int NRED = 8;                  // ring of per-tile partial row sums
constexpr int TILE = 16384;              // 128 tokens x 64 bf16, 128-byte swizzle
constexpr int AUGB = 4096;               // 128 tokens x 16 bf16 operand rows, 32-byte swizzle
constexpr long long kWaitBudget = 4000000000LL;  // clock cycles (about 2 s)
constexpr float kMaskedDual = -1e30f;    // an operand row's dual on a masked token

// nch chunks of one tile fit the ring with two to spare: chunks are reused
__host__ __device__ constexpr int nchunks(int W) { return (2 * W + 128 + 127) / 128; }
__host__ __device__ constexpr bool reuse_ok(int W) { return nchunks(W) + 2 <= NRING; }

// shared memory (offsets from a 1024-aligned base)
constexpr int OFF_A = 0;                              // 2 row-block tiles (tile parity)
constexpr int OFF_K = OFF_A + 2 * TILE;               // NRING chunk tiles
constexpr int OFF_AUG = OFF_K + NRING * TILE;         // NRING chunk operand rows
constexpr int OFF_ONES = OFF_AUG + NRING * AUGB;      // the row-block operand [1, 1, 1, 0, ...]
constexpr int OFF_WV = OFF_ONES + AUGB;               // NRING x 128 weights (WSUM)
constexpr int OFF_RED = OFF_WV + NRING * 128 * 4;     // NRED x 4 parts x 128 partial sums
// Per-tile row data, copied by the loader ahead of the epilogue (a ring of NRI
// tiles): the rows' working duals (shift sources or row duals), and the WSUM
// base and multiplier.
constexpr int NRI = 4;
struct RowInfo {
    float rw[128];
    float base[128];
    float mult[128];
};
constexpr int OFF_RI = OFF_RED + NRED * 4 * 128 * 4;
constexpr int OFF_BAR = (OFF_RI + NRI * (int)sizeof(RowInfo) + 7) / 8 * 8;
enum { B_AFULL = 0, B_AEMPTY = 2, B_FULL = 4, B_EMPTY = B_FULL + NRING, B_SFULL = B_EMPTY + NRING,
       B_SEMPTY = B_SFULL + 4, B_RFULL = B_SEMPTY + 4, B_REMPTY = B_RFULL + NRI,
       B_QFULL = B_REMPTY + NRI, B_QEMPTY = B_QFULL + NRED, B_ONES = B_QEMPTY + NRED,
       B_DRAIN = B_ONES + 1, NBAR = B_DRAIN + 1 };
constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(OFF_AUG % 1024 == 0 && OFF_ONES % 1024 == 0, "operand tiles keep the swizzle atoms aligned");

// TMA maps: row blocks (A), K chunks (B), the chunks' operand rows (BA) and
// the constant row-block operand (AO, a 128 x 16 tile)
struct Maps {
    CUtensorMap A, B, BA, AO;
};

// The constant row-block operand: 128 rows of [1, 1, 1, 0, ..., 0] (bf16 1.0 =
// 0x3F80), whose product with a chunk's operand rows adds slots 0-2 of each
// column's row, the three parts of its dual, to every score of the column.
struct OnesTile {
    uint16_t v[128 * 16];
};
constexpr OnesTile make_ones_tile() {
    OnesTile t{};
    for (int r = 0; r < 128; ++r)
        for (int k = 0; k < 3; ++k) t.v[r * 16 + k] = 0x3F80;
    return t;
}
__device__ __align__(256) const OnesTile g_aug_ones = make_ones_tile();

// Writes a token's operand row: y = dual / c as hi + mid + lo, each the bf16
// rounding of what the parts before it leave (so the three carry the 24
// significant bits of y), in slots 0-2; slots 3-15 zero.  A masked token
// (ok false) gets kMaskedDual in slot 0.
__device__ __forceinline__ void put_aug(__nv_bfloat16* dst, bool ok, float y) {
    uint32_t w0 = 0, w1 = 0;
    if (ok) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(y);
        const float r1 = y - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
        w0 = (uint32_t)__bfloat16_as_ushort(hi) | ((uint32_t)__bfloat16_as_ushort(mid) << 16);
        w1 = (uint32_t)__bfloat16_as_ushort(lo);
    } else {
        w0 = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(kMaskedDual));
    }
    uint4* o = reinterpret_cast<uint4*>(dst);
    o[0] = make_uint4(w0, w1, 0u, 0u);
    o[1] = make_uint4(0u, 0u, 0u, 0u);
}

struct Ctl {
    uint64_t* bar;
    volatile int* abort;
    int* status;
    __device__ bool wait(int slot, uint32_t parity) {
        if (tc::mbar_try_wait(bar + slot, parity)) return true;
        if (*abort) return false;
        if (tc::mbar_wait(bar + slot, parity, kWaitBudget)) return true;
        *abort = 1;
        if (status) atomicCAS(status, 0, (int)SA_ERR_TIMEOUT);
        return false;
    }
};

// (problem, row block) of the tiles of a range, advanced without divisions
struct Cursor {
    int rb, h, b;
    __device__ void next(int nb, int H) {
        if (++rb == nb) {
            rb = 0;
            if (++h == H) { h = 0; ++b; }
        }
    }
};

// Ring positions of a tile's chunks: tile `it` reads load numbers base ..
// base + nch - 1 (slot = number mod NRING).  A successor (the next row block of
// the same problem, with reuse) shares all but its last chunk with the tile
// before it.
struct ChunkIds {
    int base = 0, next = 0;
    __device__ int advance(bool successor, int nch) {  // the first chunk to load
        base = successor ? base + 1 : next;
        next = base + nch;
        return successor ? nch - 1 : 0;
    }
};

// 2^x on the FMA pipe for a pair of arguments (see the file comment); x <= 0.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& e0, float& e1) {
    const uint64_t xx = tc::pk2(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
    const uint64_t mag = tc::pk2(12582912.f, 12582912.f);  // 1.5 * 2^23
    const uint64_t t = tc::add2(xx, mag);                   // 1.5 * 2^23 + round(x)
    const uint64_t n = tc::add2(t, tc::pk2(-12582912.f, -12582912.f));
    const uint64_t f = tc::sub2(xx, n);                     // x - round(x), in [-1/2, 1/2]
    uint64_t p = tc::fma2(tc::pk2(1.327647129073739e-3f, 1.327647129073739e-3f), f,
                          tc::pk2(9.675540961325169e-3f, 9.675540961325169e-3f));
    p = tc::fma2(p, f, tc::pk2(5.550713092088699e-2f, 5.550713092088699e-2f));
    p = tc::fma2(p, f, tc::pk2(2.4022120237350464e-1f, 2.4022120237350464e-1f));
    p = tc::fma2(p, f, tc::pk2(6.931469440460205e-1f, 6.931469440460205e-1f));
    p = tc::fma2(p, f, tc::pk2(1.0000001192092896f, 1.0000001192092896f));
    float p0, p1, t0, t1;
    tc::upk2(p, p0, p1);
    tc::upk2(t, t0, t1);
    // the low bits of t hold round(x); shifted into the exponent field they add
    // round(x) to the exponent of p (the shifter's own bits shift out)
    e0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
    e1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

// One warp's 32 rows x 32 columns, staged: all arguments c2 * S' + rd (S' the
// score with the column dual folded in), then all exponentials, then the sums.
// EDGE keeps only local columns lo..hi.
template <int MODE, int KP, bool EDGE>
__device__ __forceinline__ void group(const uint32_t (&u)[32], const float* wv, uint64_t c2p,
                                      uint64_t srp, int lo, int hi, uint64_t (&acc)[4]) {
    uint64_t xp[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
        xp[j] = tc::fma2(tc::pk2(__uint_as_float(u[2 * j]), __uint_as_float(u[2 * j + 1])), c2p, srp);
    float e[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        float x0, x1;
        tc::upk2(xp[j], x0, x1);
        if (EDGE) {
            if ((unsigned)(2 * j - lo) > (unsigned)(hi - lo)) x0 = -INFINITY;
            if ((unsigned)(2 * j + 1 - lo) > (unsigned)(hi - lo)) x1 = -INFINITY;
        }
        if (!EDGE && 2 * j + 2 > 32 - KP) {
            exp2_poly2(x0, x1, e[2 * j], e[2 * j + 1]);
        } else {
            e[2 * j] = ex2(x0);
            e[2 * j + 1] = ex2(x1);
        }
    }
    if (MODE == WSUM) {
        const float4* w4 = reinterpret_cast<const float4*>(wv);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 w = w4[q];
            acc[(2 * q) & 3] = tc::fma2(tc::pk2(e[4 * q], e[4 * q + 1]), tc::pk2(w.x, w.y), acc[(2 * q) & 3]);
            acc[(2 * q + 1) & 3] = tc::fma2(tc::pk2(e[4 * q + 2], e[4 * q + 3]), tc::pk2(w.z, w.w), acc[(2 * q + 1) & 3]);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j & 3] = tc::add2(acc[j & 3], tc::pk2(e[2 * j], e[2 * j + 1]));
    }
}

template <int MODE, int KP>
__global__ void __launch_bounds__(NTHREADS, 1) tc_rowsum_sweep(const SweepArgs a,
                                                              const __grid_constant__ Maps maps,
                                                              int* status, int BH) {
    static_assert(KP % 4 == 0 && KP >= 0 && KP <= 32, "poly exponentials per group");
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint32_t* tbase = reinterpret_cast<uint32_t*>(sm + OFF_BAR + NBAR * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tbase + 1);
    float* wring = reinterpret_cast<float*>(sm + OFF_WV);
    float* red = reinterpret_cast<float*>(sm + OFF_RED);
    RowInfo* rinfo = reinterpret_cast<RowInfo*>(sm + OFF_RI);
    Ctl ctl{bar, abort_flag, status};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = a.L, W = a.W, H = a.H;
    const int nblk = (L + 127) / 128, nch = nchunks(W);
    const bool reuse = reuse_ok(W);
    // Chunk g of tile it goes to part (g + rot * it) % 4.  With nch not a
    // multiple of 4, g % 4 alone already moves a tile's chunks over the parts
    // from tile to tile; with nch a multiple of 4 it would give chunk c of every
    // tile to part c (the band-edge chunks, with fewer groups inside the band,
    // always to parts 0 and 3), so the tile index is added.
    const int rot = (nch & 3) == 0 ? 1 : 0;
    const int ntiles = BH * nblk;
    const int t0 = (int)(((long long)blockIdx.x * ntiles) / gridDim.x);
    const int t1 = (int)(((long long)(blockIdx.x + 1) * ntiles) / gridDim.x);
    const int ntl = t1 - t0;
    const Cursor cur0{t0 % nblk, (t0 / nblk) % H, (t0 / nblk) / H};

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bar + B_AFULL + i, 1);
            tc::mbar_init(bar + B_AEMPTY + i, 1);
        }
        for (int s = 0; s < NRING; ++s) {
            // the TMA bytes (+ the 32 weight lanes)
            tc::mbar_init(bar + B_FULL + s, MODE == WSUM ? 33 : 1);
            tc::mbar_init(bar + B_EMPTY + s, 1 + 4 * nch);  // the last MMA + 4 warps x nch uses
        }
        for (int b = 0; b < 4; ++b) {
            tc::mbar_init(bar + B_SFULL + b, 1);
            tc::mbar_init(bar + B_SEMPTY + b, 4);
        }
        for (int i = 0; i < NRI; ++i) {
            tc::mbar_init(bar + B_RFULL + i, 32);     // the loader lanes' copies
            tc::mbar_init(bar + B_REMPTY + i, NEPI + 1);  // every epilogue warp and the finisher
        }
        for (int i = 0; i < NRED; ++i) {
            tc::mbar_init(bar + B_QFULL + i, NEPI);   // every epilogue warp's partial row sums
            tc::mbar_init(bar + B_QEMPTY + i, 1);     // the finisher has read them
        }
        tc::mbar_init(bar + B_ONES, 1);
        tc::mbar_init(bar + B_DRAIN, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tbase, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tS = *tbase;  // score buffer b at columns 128 b
    // The set-up above overlaps the previous kernel's tail; every global
    // access comes after this wait.  Then the next sweep may begin launching:
    // its CTAs take an SM only as this grid's leave it.
    tc::grid_dep_wait();
    tc::grid_dep_launch();

    if (warp == W_LOAD) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            tc::prefetch_tmap(&maps.A);
            tc::prefetch_tmap(&maps.B);
            tc::prefetch_tmap(&maps.BA);
            tc::prefetch_tmap(&maps.AO);
            tc::mbar_expect_tx(bar + B_ONES, AUGB);
            tc::tma_load_3d(sm + OFF_ONES, &maps.AO, bar + B_ONES, 0, 0, 0);
        }
        ChunkIds ids;
        int issued = 0, a_issued = 0, pbh = -1, prb = -1;
        bool ok = true;
        Cursor cur = cur0;
        for (int it = 0; ok && it < ntl; ++it, cur.next(nblk, H)) {
            const int bh = cur.b * H + cur.h, r0 = cur.rb * 128;
            const bool succ = reuse && bh == pbh && cur.rb == prb + 1;
            pbh = bh;
            prb = cur.rb;
            const int first = ids.advance(succ, nch);
            if (lane == 0) {
                if (it >= 2 && !ctl.wait(B_AEMPTY + (it & 1), ((it >> 1) - 1) & 1)) ok = false;
                if (ok && SA_BOUNDS(bh < BH && r0 >= 0 && r0 < L, status)) {
                    tc::mbar_expect_tx(bar + B_AFULL + (it & 1), TILE);
                    tc::tma_load_3d(sm + OFF_A + (it & 1) * TILE, &maps.A, bar + B_AFULL + (it & 1), 0,
                                    r0, bh);
                    a_issued = it + 1;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            // the tile's row data (lane l copies rows 32k + l)
            if (ok && it >= NRI && !ctl.wait(B_REMPTY + it % NRI, ((it / NRI) - 1) & 1)) ok = false;
            if (ok) {
                RowInfo& ri = rinfo[it % NRI];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int r = r0 + 32 * k + lane;
                    const bool in = r < L;
                    const long long o = (long long)bh * a.rdw.s + (in ? r : 0);
                    tc::cp_async4(&ri.rw[32 * k + lane], a.rdw.p + o, in);
                    if (MODE == WSUM) {
                        const long long ob = (long long)bh * a.base.s + (in ? r : 0);
                        const long long om = (long long)bh * a.mult.s + (in ? r : 0);
                        tc::cp_async4(&ri.base[32 * k + lane], a.base.p ? a.base.p + ob : a.rdw.p + o,
                                      in && a.base.p);
                        tc::cp_async4(&ri.mult[32 * k + lane], a.mult.p ? a.mult.p + om : a.rdw.p + o,
                                      in && a.mult.p);
                    }
                }
                tc::cp_async_arrive(bar + B_RFULL + it % NRI);
            }
            for (int c = first; ok && c < nch; ++c) {
                const int id = ids.base + c, s = id % NRING;
                if (id >= NRING && !ctl.wait(B_EMPTY + s, ((id / NRING) - 1) & 1)) { ok = false; break; }
                const int col0 = r0 - W + 128 * c;
                if (lane == 0 && SA_BOUNDS(s < NRING && col0 >= -W - 128 && col0 < L + W + 128, status)) {
                    tc::mbar_expect_tx(bar + B_FULL + s, TILE + AUGB);
                    tc::tma_load_3d(sm + OFF_K + s * TILE, &maps.B, bar + B_FULL + s, 0, col0, bh);
                    tc::tma_load_3d(sm + OFF_AUG + s * AUGB, &maps.BA, bar + B_FULL + s, 0, col0, bh);
                    // The slot is released once every tile that reads the chunk has
                    // (each use arrives 4 times, the last use's MMA once): the uses
                    // are this tile and the successors that follow it, at most c of
                    // them; the uses that will not happen are arrived for here.
                    int uses = 1;
                    if (reuse) {
                        Cursor ln = cur;
                        int pb = bh, pr = cur.rb;
                        for (int k = 1; k <= c && it + k < ntl; ++k) {
                            ln.next(nblk, H);
                            if (ln.b * H + ln.h != pb || ln.rb != pr + 1) break;
                            pr = ln.rb;
                            ++uses;
                        }
                    }
                    if (uses < nch) tc::mbar_arrive_cnt(bar + B_EMPTY + s, 4 * (nch - uses));
                }
                issued = id + 1;
                if (MODE == WSUM) {  // the weights, zero off [0, L)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int col = col0 + 32 * k + lane;
                        const bool in = col >= 0 && col < L;
                        tc::cp_async4(&wring[s * 128 + 32 * k + lane],
                                      a.w.p + (long long)bh * a.w.s + (in ? col : 0), in);
                    }
                    tc::cp_async_arrive(bar + B_FULL + s);
                }
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");  // nothing in flight at exit
        if (lane == 0) {  // let issued loads land before teardown
            tc::mbar_wait(bar + B_ONES, 0, kWaitBudget);
            if (*abort_flag) {
                for (int x = max(0, a_issued - 2); x < a_issued; ++x)
                    tc::mbar_wait(bar + B_AFULL + (x & 1), (x >> 1) & 1, kWaitBudget);
                for (int x = max(0, issued - NRING); x < issued; ++x)
                    tc::mbar_wait(bar + B_FULL + x % NRING, (x / NRING) & 1, kWaitBudget);
            }
        }
        __syncwarp();
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop (uniform control flow and values); one
        // elected lane issues the MMAs and commits.  A chunk's scores are four
        // K16 steps of Q K^T and a fifth that adds the column duals.
        const uint32_t id_s = tc::idesc_bf16(128, 128, false, false);
        const uint64_t dA0 = tc::sdesc_sw128(tc::smem_u32(sm + OFF_A), 16, 1024);
        const uint64_t dK0 = tc::sdesc_sw128(tc::smem_u32(sm + OFF_K), 16, 1024);
        const uint64_t dOnes = tc::sdesc_sw32(tc::smem_u32(sm + OFF_ONES));
        const uint64_t dAug0 = tc::sdesc_sw32(tc::smem_u32(sm + OFF_AUG));
        ChunkIds ids;
        int g = 0, pbh = -1, prb = -1;
        int nb[4] = {0, 0, 0, 0};  // uses of each TMEM buffer so far
        bool ok = ctl.wait(B_ONES, 0);
        Cursor cur = cur0;
        for (int it = 0; ok && it < ntl; ++it) {
            const int bh = cur.b * H + cur.h;
            const bool succ = reuse && bh == pbh && cur.rb == prb + 1;
            pbh = bh;
            prb = cur.rb;
            ids.advance(succ, nch);
            Cursor nx = cur;
            nx.next(nblk, H);
            const bool next_succ = reuse && it + 1 < ntl && nx.b * H + nx.h == bh && nx.rb == cur.rb + 1;
            if (!ctl.wait(B_AFULL + (it & 1), (it >> 1) & 1)) { ok = false; break; }
            const uint64_t dA = tc::sdesc_add(dA0, (it & 1) * TILE);
            for (int c = 0; c < nch; ++c, ++g) {
                // buffer = the part that processes the chunk (see the epilogue)
                const int id = ids.base + c, s = id % NRING, b = (g + rot * it) & 3;
                const int u = b == 0 ? nb[0] : b == 1 ? nb[1] : b == 2 ? nb[2] : nb[3];
                if (!ctl.wait(B_FULL + s, (id / NRING) & 1)) { ok = false; break; }
                if (u >= 1 && !ctl.wait(B_SEMPTY + b, (u - 1) & 1)) { ok = false; break; }
                if (b == 0) ++nb[0]; else if (b == 1) ++nb[1]; else if (b == 2) ++nb[2]; else ++nb[3];
                tc::tc_fence_after();
                const uint64_t dB = tc::sdesc_add(dK0, s * TILE);
                if (tc::elect_one()) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_bf16(tS + 128 * b, tc::sdesc_add(dA, 32 * k), tc::sdesc_add(dB, 32 * k),
                                     id_s, k > 0);
                    tc::mma_bf16(tS + 128 * b, dOnes, tc::sdesc_add(dAug0, s * AUGB), id_s, 1u);
                    tc::tc_commit(bar + B_SFULL + b);
                    if (!next_succ || c == 0) tc::tc_commit(bar + B_EMPTY + s);  // its last reader
                }
                __syncwarp();
            }
            if (!ok) break;
            if (tc::elect_one()) tc::tc_commit(bar + B_AEMPTY + (it & 1));
            __syncwarp();
            cur = nx;
        }
        if (tc::elect_one()) tc::tc_commit(bar + B_DRAIN);
        __syncwarp();
        tc::mbar_wait(bar + B_DRAIN, 0, kWaitBudget);
    } else if (warp == W_FIN) {
        // ------------------------------------------------------------ finisher
        // Each tile's outputs from the four parts' partial row sums; lane l
        // writes rows 32k + l.  An LSE sweep also writes its output's working
        // copy and operand row for the sweep after it.
        const float inv_c2 = 1.f / a.c2;
        Cursor cur = cur0;
        for (int it = 0; it < ntl; ++it, cur.next(nblk, H)) {
            const int bh = cur.b * H + cur.h, r0 = cur.rb * 128, slot = it % NRED;
            if (!ctl.wait(B_RFULL + it % NRI, (it / NRI) & 1)) break;
            if (!ctl.wait(B_QFULL + slot, (it / NRED) & 1)) break;
            const RowInfo& ri = rinfo[it % NRI];
            const float* rs = red + slot * 512;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int lr = 32 * k + lane, r = r0 + lr;
                const float rwv = ri.rw[lr];
                const bool valid = r < L && rwv != -INFINITY;
                const float tot = (rs[lr] + rs[128 + lr]) + (rs[256 + lr] + rs[384 + lr]);
                if (r < L && SA_BOUNDS(bh < BH, status)) {
                    float out = 0.f, outw = -INFINITY;
                    if (valid) {
                        if (MODE == LSE) {
                            outw = rwv - lg2(tot);
                            out = outw * kLn2;
                        } else {
                            const float bb = ri.base[lr];
                            const float mu = a.mult.p ? ri.mult[lr] : 1.f;
                            out = bb + a.sgn * mu * tot;
                        }
                    }
                    a.out_vec.at(bh, r) = out;
                    if (MODE == LSE && a.outw.p) a.outw.at(bh, r) = outw;
                    if (MODE == LSE && a.augo)
                        put_aug(reinterpret_cast<__nv_bfloat16*>(a.augo) + (long long)bh * a.aug_s + 16LL * r,
                                valid, outw * inv_c2);
                }
            }
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(bar + B_QEMPTY + slot);
                tc::mbar_arrive(bar + B_REMPTY + it % NRI);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int qd = warp & 3, pt = warp >> 2;
        const uint32_t lanebase = (uint32_t)(qd * 32) << 16;
        const uint64_t c2p = tc::pk2(a.c2, a.c2);
        ChunkIds ids;
        int g = 0, pbh = -1, prb = -1;
        int nu = 0;  // chunks this part has processed (uses of its TMEM buffer)
        bool ok = true;
        Cursor cur = cur0;
        for (int it = 0; ok && it < ntl; ++it) {
            const int bh = cur.b * H + cur.h, r0 = cur.rb * 128;
            const bool succ = reuse && bh == pbh && cur.rb == prb + 1;
            pbh = bh;
            prb = cur.rb;
            ids.advance(succ, nch);
            Cursor nx = cur;
            nx.next(nblk, H);
            // this thread's row and its shift (its working dual; -inf on an
            // invalid row, whose sum is not used)
            const int rw0 = r0 + qd * 32, r = rw0 + lane;
            if (!ctl.wait(B_RFULL + it % NRI, (it / NRI) & 1)) { ok = false; break; }
            const float rwv = rinfo[it % NRI].rw[qd * 32 + lane];
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar + B_REMPTY + it % NRI);
            const float sr = r < L ? rwv : -INFINITY;
            const uint64_t srp = tc::pk2(sr, sr);
            uint64_t acc[4] = {0, 0, 0, 0};
            // this part's chunks of the tile: c = c0, c0 + 4, ...; chunk g_t + c
            // goes to part (g_t + c + rot * it) % 4, in that part's own TMEM
            // buffer, whose phases its one part consumes in order
            const int g_t = g;
            g += nch;
            for (int c = (pt - (g_t + rot * it)) & 3; c < nch; c += 4) {
                const int id = ids.base + c, s = id % NRING, b = pt;
                if (!ctl.wait(B_SFULL + b, nu & 1)) { ok = false; break; }
                ++nu;
                if (MODE == WSUM && !ctl.wait(B_FULL + s, (id / NRING) & 1)) { ok = false; break; }
                tc::tc_fence_after();
                const int col0 = r0 - W + 128 * c;
                const float* wv = wring + s * 128;
#pragma unroll 1
                for (int gr = 0; gr < 4; ++gr) {
                    const int cg = col0 + 32 * gr;
                    const bool all_out = (cg + 31 < rw0 - W) || (cg > rw0 + 31 + W) || cg + 31 < 0 || cg >= L;
                    if (all_out) continue;
                    const bool all_in = (cg >= rw0 + 31 - W) && (cg + 31 <= rw0 + W) && cg >= 0 && cg + 31 < L;
                    uint32_t u[32];
                    if (SA_BOUNDS(128 * b + 32 * gr + 32 <= 512, status))
                        tc::tmem_ld32(tS + 128 * b + lanebase + 32 * gr, u);
                    tc::tmem_wait_ld();
                    const float* ws = wv + 32 * gr;
                    // this row's band and [0, L), as local columns of the group
                    const int lo = max(r - W, 0) - cg, hi = min(r + W, L - 1) - cg;
                    if (all_in) group<MODE, KP, false>(u, ws, c2p, srp, lo, hi, acc);
                    else group<MODE, KP, true>(u, ws, c2p, srp, lo, hi, acc);
                }
                // every TMEM read and shared-memory read of the chunk is done
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    tc::mbar_arrive(bar + B_SEMPTY + b);
                    tc::mbar_arrive(bar + B_EMPTY + s);  // this use has read the slot
                }
            }
            if (!ok) break;
            // ---------------------------------------------------------- end of tile
            // this part's partial row sums, for the finisher
            float a0, a1, a2, a3, a4, a5, a6, a7;
            tc::upk2(acc[0], a0, a1);
            tc::upk2(acc[1], a2, a3);
            tc::upk2(acc[2], a4, a5);
            tc::upk2(acc[3], a6, a7);
            const int slot = it % NRED;
            if (it >= NRED && !ctl.wait(B_QEMPTY + slot, ((it / NRED) - 1) & 1)) { ok = false; break; }
            if (SA_BOUNDS(slot < NRED && pt < 4, status))
                red[slot * 512 + pt * 128 + qd * 32 + lane] = ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar + B_QFULL + slot);
            cur = nx;
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tS, 512);
    }
}

}  // namespace tcr
}  // namespace sa
