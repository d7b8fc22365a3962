// One Sinkhorn iteration (row update and column update) in one pass over the
// band, on the tensor cores.  bf16 storage, band half-width W <= 256.
//
// Iteration k turns (u_{k-1}, v_{k-1}) into u_k and the column sums that
// define v_k.  For a block of 128 rows i and its 2W+128 columns j:
//   E_ij  = exp(S_ij + u_{k-1,i} + v_{k-1,j})   (<= 1: v_{k-1} normalised the
//                                               columns of exp(S + u_{k-1} + v))
//   r_i   = sum_j E_ij,    u_k,i = u_{k-1,i} - log r_i
//   part_j = sum_i E_ij / r_i   (= exp(-v_{k-1,j}) sum_i exp(S_ij + u_k,i))
// and v_k,j = v_{k-1,j} - log(sum over the row blocks covering j of part_j),
// which the next iteration (or the final reduction) forms.  So each band entry
// costs one exponential per iteration instead of two.  A column is covered by
// at most 6 row blocks (W <= 256); their partials sit in 8 slots per column,
// slot = row block mod 8, so a column's partials are 32 contiguous bytes and are
// always summed in the same order.
//
// The row sums stay in registers.  The column sums are a contraction over the
// rows, done on the tensor core: E is rounded to fp16 and staged in shared
// memory (one 128 x 128 tile per column chunk, 128-byte swizzle); once r is
// known the MMA computes D[j, n] = sum_i E[i, j] w[i, n], where w holds 1/r of
// the rows of quadrant q (rows 32q..32q+31) in columns n = 2q (fp16 high part)
// and 2q+1 (low part), scaled by the quadrant's largest 1/r.
//
// Persistent CTAs (one per SM) each walk a contiguous range of (batch*head,
// row block) tiles, so consecutive tiles of a range share all but one column
// chunk: the column duals of a chunk are formed once and kept in a ring of
// chunk slots.  The chunks of the range are numbered g = 0, 1, ...; the score
// tile of chunk g sits in TMEM buffer g mod 2 and is consumed by epilogue group
// g mod 2 (8 warps: each thread one row, each warp 64 of the 128 columns), so
// the two groups work on neighbouring chunks of the same tile.  Per row
// quadrant, the warp of part 0 adds the other parts' row sums and forms u, 1/r
// and the quadrant's scale.  Warp roles: warps 0-15 epilogue (lane quadrant
// w%4, part w/4 = 2 * group + column half), warp 16 TMA loader (Q blocks, K
// chunks), warp 17 score MMAs, warp 18 column-sum MMAs (issued apart so that
// score tiles never queue behind them), warp 19 column and row duals.  Every
// mbarrier wait is bounded.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace sa {
namespace tcf {

constexpr int NEPI = 16;           // epilogue warps: lane quadrant (w % 4) x part (w / 4)
constexpr int NQ = NEPI / 4;       // parts per quadrant
constexpr int W_LOAD = NEPI, W_MMA = NEPI + 1, W_COL = NEPI + 2, W_CV = NEPI + 3;
constexpr int NTHREADS = (NEPI + 4) * 32;
constexpr int NSLOT = 8;           // partial slots per column
constexpr int TILE = 16384;        // 128 x 64 bf16 (or 128 x 64 fp16) swizzled tile
constexpr int NST = 2;             // K-chunk stages
constexpr int MAXCH = 5;           // column chunks per row block (2W + 128 <= 640)
constexpr int NCVS = 2 * MAXCH;    // column-dual chunk slots
constexpr int NWM = 3;             // ring of per-tile quadrant scales
constexpr long long kWaitBudget = 4000000000LL;

// shared-memory carve-up (from a 1024-aligned base)
constexpr int OFF_A = 0;
constexpr int OFF_STAGE = TILE;
constexpr int OFF_E = OFF_STAGE + NST * TILE;
constexpr int OFF_W = OFF_E + MAXCH * 2 * TILE;  // 16 x 128 fp16, two 2 KB K-blocks
constexpr int OFF_CV = OFF_W + 4096;             // NCVS x 128 floats
constexpr int OFF_ROW = OFF_CV + NCVS * 128 * 4; // 2 x 128 row duals (log2 units)
constexpr int OFF_RED = OFF_ROW + 2 * 128 * 4;   // 2 x (4 quadrants x 4 parts x 32) floats
constexpr int OFF_WM = OFF_RED + 2 * 512 * 4;    // NWM x 4 floats
constexpr int OFF_BAR = OFF_WM + 64;
constexpr int SMEM_BYTES = OFF_BAR + 32 * 8 + 16 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

enum { B_AFULL = 0, B_AEMPTY = 1, B_FULL = 2, B_EMPTY = 4, B_SFULL = 6, B_SEMPTY = 8,
       B_CVFULL = 10, B_CVEMPTY = 12, B_WFULL = 14, B_DRAIN = 15, B_DRAIN2 = 16,
       B_QF = 17 /* .. 20: a quadrant's three partial row sums written */,
       B_QE = 21 /* .. 24: a quadrant's row sums read */,
       B_CS = 25 /* .. 25 + MAXCH - 1: column sums of chunk c done */ };
static_assert(B_CS + MAXCH <= 32, "barrier slots");

struct FusedArgs {
    int L, W, H, BH, nblk, ncol, nch;  // ncol = 2W + 128, nch = ceil(ncol / 128)
    float c2;                          // score scale * log2(e)
    const uint8_t* mask;               // [B][L] or null
    Vec u_prev;                        // u_{k-1}
    MVec u_out;                        // u_k (may alias u_prev)
    Vec v_src;                         // v_{k-1} (materialised) or v_{k-2} (with part_in)
    MVec v_out;                        // with part_in: v_{k-1} (each column written once)
    const float* part_in;              // column partials of v_{k-1}, or null
    float* part_out;                   // column partials of v_k: [BH][L][NSLOT]
    int* status;
};

__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}

// This CTA's contiguous tile range [t0, t1).
__device__ __forceinline__ void tile_range(int ntiles, int& t0, int& t1) {
    t0 = (int)(((long long)blockIdx.x * ntiles) / gridDim.x);
    t1 = (int)(((long long)(blockIdx.x + 1) * ntiles) / gridDim.x);
}

// Column-dual chunk ids: tile `it` of a range uses ids base .. base + nch - 1
// (slot = id mod NCVS).  A tile that follows its predecessor's row block in the
// same (batch, head) shares all but its last chunk with it.
struct ChunkIds {
    int base = 0, next = 0;
    __device__ int advance(bool successor, int nch) {  // returns the first new chunk
        const int first_new = successor ? nch - 1 : 0;
        base = successor ? base + 1 : next;
        next = base + nch;
        return first_new;
    }
};

struct Ctl {
    uint64_t* bar;
    volatile int* abort;
    int* status;
    __device__ bool wait(int slot, uint32_t parity) {
        if (tc::mbar_try_wait(bar + slot, parity)) return true;  // complete: no abort check
        if (*abort) return false;
        if (tc::mbar_wait(bar + slot, parity, kWaitBudget)) return true;
        *abort = 1;
        if (status) atomicCAS(status, 0, (int)SA_ERR_TIMEOUT);
        return false;
    }
};

// Sum of the partials of column `col` over the row blocks that cover it
// (slot s holds row block lo + ((s - lo) mod 8) when that is <= hi), in slot
// order, so every CTA forms the same value.
__device__ __forceinline__ float partial_sum(const FusedArgs& a, int col, float4 p0, float4 p1) {
    const int x = col - 127 - a.W;
    const int lo = x <= 0 ? 0 : (x + 127) / 128;
    const int hi = min(a.nblk - 1, (col + a.W) / 128);
    const float sl[NSLOT] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < NSLOT; ++i)
        if (lo + ((i - lo) & (NSLOT - 1)) <= hi) sum += sl[i];
    return sum;
}

// v_{k-1} of column `col` from v_{k-2} and the covering row blocks' partials.
__device__ __forceinline__ float v_from_partials(const FusedArgs& a, int bh, int col) {
    const float4* p = reinterpret_cast<const float4*>(a.part_in + ((size_t)bh * a.L + col) * NSLOT);
    return a.v_src.at(bh, col) - lg2(partial_sum(a, col, p[0], p[1])) * kLn2;
}

// E = exp2(c2 * s + cv + rd2) for one thread's 32 columns, packed to fp16
// pairs in `ep`; `CHECK` masks the entries off the band (only the groups that
// straddle the band's edge).  The fp32 values are added to two packed pairs of
// row-sum accumulators (columns 4q, 4q + 1 into acc[0]; 4q + 2, 4q + 3 into acc[1]).
template <bool CHECK>
__device__ __forceinline__ void group_exp(const uint32_t (&u)[32], const float* cvp, float c2, float rd2,
                                          int d_first, int W, uint32_t (&ep)[16], uint64_t (&acc)[2]) {
    const float4* c4 = reinterpret_cast<const float4*>(cvp);
    const uint64_t c2p = tc::pk2(c2, c2), rdp = tc::pk2(rd2, rd2);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 cvv = c4[q];
        float x0, x1, x2, x3;
        tc::upk2(tc::fma2(tc::pk2(__uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1])), c2p,
                          tc::add2(tc::pk2(cvv.x, cvv.y), rdp)), x0, x1);
        tc::upk2(tc::fma2(tc::pk2(__uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3])), c2p,
                          tc::add2(tc::pk2(cvv.z, cvv.w), rdp)), x2, x3);
        if (CHECK) {
            const int d0 = d_first - 4 * q;  // row - column of element 4q
            if ((unsigned)(d0 + W) > (unsigned)(2 * W)) x0 = -INFINITY;
            if ((unsigned)(d0 - 1 + W) > (unsigned)(2 * W)) x1 = -INFINITY;
            if ((unsigned)(d0 - 2 + W) > (unsigned)(2 * W)) x2 = -INFINITY;
            if ((unsigned)(d0 - 3 + W) > (unsigned)(2 * W)) x3 = -INFINITY;
        }
        const float e0 = ex2(x0), e1 = ex2(x1), e2 = ex2(x2), e3 = ex2(x3);
        acc[0] = tc::add2(acc[0], tc::pk2(e0, e1));
        acc[1] = tc::add2(acc[1], tc::pk2(e2, e3));
        ep[2 * q] = pack_f16(e0, e1);
        ep[2 * q + 1] = pack_f16(e2, e3);
    }
}

// One warp forms 128 column duals of chunk `cb` of the tile at row block r0 of
// problem bh into `cv` (v * log2(e) on valid columns, -inf outside [0, L) and on
// masked columns; entries of a chunk outside the tile's band are masked by the
// epilogue, so a column's value does not depend on the tile), and with
// `do_rows` the tile's 128 row duals into `rows` (log2 units, -inf on rows past
// L or masked).  Every load is issued before any value is used.  v_{k-1} of a
// column is written to v_out by the CTA whose range [t0, t1) holds the column's
// own row block.
__device__ __forceinline__ void dual_batch(const FusedArgs& a, int bh, int r0, const uint8_t* mk_,
                                           int cb, bool do_cols, bool do_rows, float* cv, float* rows,
                                           int t0, int t1, int lane) {
    const int L = a.L, W = a.W;
    float4 p0[4], p1[4];
    float vs[4], ur[4];
    bool inr[4], mok[4], rin[4], rmk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int cc = cb * 128 + 32 * k + lane, col = r0 - W + cc;
        inr[k] = do_cols && col >= 0 && col < L;
        mok[k] = true;
        vs[k] = 0.f;
        p0[k] = p1[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (inr[k]) {
            if (mk_) mok[k] = mk_[col] != 0;
            vs[k] = a.v_src.at(bh, col);
            if (a.part_in) {
                const float4* pp = reinterpret_cast<const float4*>(a.part_in + ((size_t)bh * L + col) * NSLOT);
                p0[k] = pp[0];
                p1[k] = pp[1];
            }
        }
        const int r = r0 + 32 * k + lane;
        rin[k] = do_rows && r < L;
        rmk[k] = true;
        ur[k] = 0.f;
        if (rin[k]) {
            if (mk_) rmk[k] = mk_[r] != 0;
            ur[k] = a.u_prev.at(bh, r);
        }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if (do_cols) {
            const int cc = cb * 128 + 32 * k + lane, col = r0 - W + cc;
            const bool valid = inr[k] && mok[k];
            float v = vs[k];
            if (a.part_in) v -= lg2(partial_sum(a, col, p0[k], p1[k])) * kLn2;
            if (a.part_in && a.v_out.p && inr[k]) {
                const int owner = bh * a.nblk + col / 128;
                if (owner >= t0 && owner < t1) a.v_out.at(bh, col) = valid ? v : 0.f;
            }
            cv[32 * k + lane] = valid ? v * kLog2e : -INFINITY;
        }
        if (do_rows) rows[32 * k + lane] = (rin[k] && rmk[k]) ? ur[k] * kLog2e : -INFINITY;
    }
}

__global__ void __launch_bounds__(NTHREADS, 1) tc_fused_iter(const FusedArgs a,
                                                            const __grid_constant__ CUtensorMap mq,
                                                            const __grid_constant__ CUtensorMap mk) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint32_t* tbase = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 32 * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tbase + 1);
    float* cvring = reinterpret_cast<float*>(sm + OFF_CV);
    float* rowring = reinterpret_cast<float*>(sm + OFF_ROW);
    float* red = reinterpret_cast<float*>(sm + OFF_RED);
    float* wmring = reinterpret_cast<float*>(sm + OFF_WM);
    Ctl ctl{bar, abort_flag, a.status};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = a.L, W = a.W, nch = a.nch, nblk = a.nblk;
    int t0, t1;
    tile_range(a.BH * nblk, t0, t1);
    const int ntl = t1 - t0;

    // zero the 1/r operand once (each quadrant only ever writes its own rows
    // of its own two columns)
    for (int t = threadIdx.x; t < 4096 / 16; t += NTHREADS)
        reinterpret_cast<uint4*>(sm + OFF_W)[t] = make_uint4(0, 0, 0, 0);
    tc::fence_async_smem();
    if (threadIdx.x == 0) {
        tc::mbar_init(bar + B_AFULL, 1);
        tc::mbar_init(bar + B_AEMPTY, 1);
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bar + B_FULL + i, 1);
            tc::mbar_init(bar + B_EMPTY + i, 1);
            tc::mbar_init(bar + B_CVFULL + i, 32);
            tc::mbar_init(bar + B_CVEMPTY + i, NEPI);
            tc::mbar_init(bar + B_SFULL + i, 1);
            tc::mbar_init(bar + B_SEMPTY + i, NEPI / 2);
        }
        for (int q = 0; q < 4; ++q) {
            tc::mbar_init(bar + B_QF + q, NQ - 1);
            tc::mbar_init(bar + B_QE + q, 1);
        }
        tc::mbar_init(bar + B_WFULL, NEPI);
        for (int c = 0; c < MAXCH; ++c) tc::mbar_init(bar + B_CS + c, 1);
        tc::mbar_init(bar + B_DRAIN, 1);
        tc::mbar_init(bar + B_DRAIN2, 1);
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
    const uint32_t tm = *tbase;
    // TMEM: score buffers at columns 0 and 128; column sums of chunk c at 256 + 32c
    // (even K steps) and 256 + 32c + 16 (odd K steps)
    const uint32_t tS = tm, tD = tm + 256;

    // the first tile's duals (all its chunks at once), by warps 0..nch-1 and
    // the last epilogue warp for the rows; ring slots 0..nch-1
    if (ntl >= 1 && (warp < nch || warp == NEPI - 1)) {
        const int bh = t0 / nblk, r0 = (t0 % nblk) * 128;
        const uint8_t* mk_ = a.mask ? a.mask + (size_t)(bh / a.H) * L : nullptr;
        dual_batch(a, bh, r0, mk_, warp, warp < nch, warp == NEPI - 1, cvring + warp * 128,
                   rowring, t0, t1, lane);
    }
    __syncthreads();

    if (warp == W_CV) {
        // ------------------------------------------------------------ column and row duals
        ChunkIds ids;
        for (int it = 0; it < ntl; ++it) {
            const int t = t0 + it, bh = t / nblk, rb = t % nblk, r0 = rb * 128;
            const uint8_t* mk_ = a.mask ? a.mask + (size_t)(bh / a.H) * L : nullptr;
            const int first = ids.advance(it > 0 && rb > 0, nch);
            if (it >= 2 && !ctl.wait(B_CVEMPTY + (it & 1), ((it >> 1) - 1) & 1)) break;
            // Per batch of 128 columns, every load is issued before any value is
            // used.  The tile's row duals (log2 units, -inf on rows past L or
            // masked) come with the first batch; a tile's rows are written only
            // at the end of that tile.
            if (it >= 1)  // tile 0's duals were formed by every warp before the roles split
                for (int cb = first; cb < nch; ++cb)
                    dual_batch(a, bh, r0, mk_, cb, true, cb == first,
                               cvring + ((ids.base + cb) % NCVS) * 128, rowring + (it & 1) * 128,
                               t0, t1, lane);
            tc::mbar_arrive(bar + B_CVFULL + (it & 1));
        }
    } else if (warp == W_LOAD) {
        // ------------------------------------------------------------ TMA loader
        if (lane == 0) {
            int g = 0, issued = 0;
            bool ok = true;
            for (int it = 0; ok && it < ntl; ++it) {
                const int t = t0 + it, bh = t / nblk, r0 = (t % nblk) * 128;
                if (it >= 1 && !ctl.wait(B_AEMPTY, (it - 1) & 1)) break;
                tc::mbar_expect_tx(bar + B_AFULL, TILE);
                tc::tma_load_3d(sm + OFF_A, &mq, bar + B_AFULL, 0, r0, bh);
                for (int c = 0; ok && c < nch; ++c, ++g) {
                    const int s = g % NST;
                    if (g >= NST && !ctl.wait(B_EMPTY + s, ((g / NST) - 1) & 1)) { ok = false; break; }
                    tc::mbar_expect_tx(bar + B_FULL + s, TILE);
                    tc::tma_load_3d(sm + OFF_STAGE + s * TILE, &mk, bar + B_FULL + s, 0,
                                    r0 - W + 128 * c, bh);
                    issued = g + 1;
                }
            }
            if (*abort_flag) {  // let issued loads land before teardown
                for (int x = max(0, issued - NST); x < issued; ++x)
                    tc::mbar_wait(bar + B_FULL + x % NST, (x / NST) & 1, kWaitBudget);
            }
        }
        __syncwarp();
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ score MMAs
        if (lane == 0) {
            const uint32_t id_s = tc::idesc_bf16(128, 128, false, false);
            // descriptors built once; offsets are added in 16-byte units
            const uint64_t dA = tc::sdesc_sw128(tc::smem_u32(sm + OFF_A), 16, 1024);
            const uint64_t dSt = tc::sdesc_sw128(tc::smem_u32(sm + OFF_STAGE), 16, 1024);
            bool ok = true;
            int g = 0;
            for (int it = 0; ok && it < ntl; ++it) {
                if (!ctl.wait(B_AFULL, it & 1)) { ok = false; break; }
                for (int c = 0; c < nch; ++c, ++g) {
                    const int s = g % NST, b = g & 1;
                    if (!ctl.wait(B_FULL + s, (g / NST) & 1)) { ok = false; break; }
                    if (g >= 2 && !ctl.wait(B_SEMPTY + b, ((g >> 1) - 1) & 1)) { ok = false; break; }
                    tc::tc_fence_after();
                    const uint64_t dB = tc::sdesc_add(dSt, s * TILE);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_bf16(tS + 128 * b, tc::sdesc_add(dA, 32 * k), tc::sdesc_add(dB, 32 * k),
                                     id_s, k > 0);
                    tc::tc_commit(bar + B_SFULL + b);
                    tc::tc_commit(bar + B_EMPTY + s);
                }
                if (!ok) break;
                tc::tc_commit(bar + B_AEMPTY);
            }
            tc::tc_commit(bar + B_DRAIN);
            tc::mbar_wait(bar + B_DRAIN, 0, kWaitBudget);
        }
        __syncwarp();
    } else if (warp == W_COL) {
        // ------------------------------------------------------------ column-sum MMAs
        // D[j, n] = sum_i E[i, j] w[i, n] of each tile once its row sums are
        // known; chunk c's commit frees its E tile.
        if (lane == 0) {
            const uint32_t id_c = idesc_f16(128, 16, true, false);
            const uint64_t dE = tc::sdesc_sw128(tc::smem_u32(sm + OFF_E), TILE, 1024);
            uint64_t dW[8];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                dW[kk] = tc::sdesc_sw128(tc::smem_u32(sm + OFF_W) + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);
            for (int it = 0; it < ntl; ++it) {
                if (!ctl.wait(B_WFULL, it & 1)) break;
                tc::tc_fence_after();
                for (int c = 0; c < nch; ++c) {
                    const uint64_t dEc = tc::sdesc_add(dE, c * 2 * TILE);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_bf16(tD + 32 * c + 16 * (kk & 1), tc::sdesc_add(dEc, kk * 2048), dW[kk],
                                     id_c, kk > 1);
                    tc::tc_commit(bar + B_CS + c);
                }
            }
            tc::tc_commit(bar + B_DRAIN2);
            tc::mbar_wait(bar + B_DRAIN2, 0, kWaitBudget);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int qd = warp & 3, pt = warp >> 2, grp = pt >> 1, hf = pt & 1;
        const int lr = qd * 32 + lane;
        const uint32_t lanebase = (uint32_t)(qd * 32) << 16;
        const float c2 = a.c2;
        ChunkIds ids;
        // partial of column 128c + lr of tile it_prev (problem pbh, row block prb),
        // from its two accumulators in TMEM (complete) and the quadrant scales
        auto put_partial = [&](int it_prev, int pbh, int prb, int c) {
            uint32_t d0[8], d1[8];
            tmem_ld8(tD + lanebase + 32 * c, d0);
            tmem_ld8(tD + lanebase + 32 * c + 16, d1);
            tc::tmem_wait_ld();
            const float* wm = wmring + (it_prev % NWM) * 4;
            float s = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                s = fmaf(wm[q], (__uint_as_float(d0[2 * q]) + __uint_as_float(d0[2 * q + 1])) +
                                    (__uint_as_float(d1[2 * q]) + __uint_as_float(d1[2 * q + 1])), s);
            const int cc = 128 * c + lr, col = prb * 128 - W + cc;
            if (cc < a.ncol && col >= 0 && col < L)
                a.part_out[((size_t)pbh * L + col) * NSLOT + (prb & (NSLOT - 1))] = s;
        };
        bool ok = true;
        // (problem, row block) of tile t0 + it, advanced without divisions, and
        // of the tile before it
        int bh = t0 / nblk, rb = t0 % nblk, pbh = 0, prb = 0;
        for (int it = 0; ok && it < ntl; ++it) {
            if (it > 0) {
                pbh = bh;
                prb = rb;
                if (++rb == nblk) { rb = 0; ++bh; }
            }
            const int r0 = rb * 128;
            const int r = r0 + lr, rw0 = r0 + qd * 32;
            ids.advance(it > 0 && rb > 0, nch);
            if (!ctl.wait(B_CVFULL + (it & 1), (it >> 1) & 1)) { ok = false; break; }
            // invalid rows carry -inf: all their E are 0
            const float rd2 = rowring[(it & 1) * 128 + lr];
            const bool rok = rd2 != -INFINITY;
            uint64_t acc4[2] = {0, 0};  // partial row sums, packed pairs
            for (int c = 0; c < nch; ++c) {
                const int g = it * nch + c, b = g & 1;
                if (b != grp) continue;  // the other group's chunk
                if (!ctl.wait(B_SFULL + b, (g >> 1) & 1)) { ok = false; break; }
                const float* cvc = cvring + ((ids.base + c) % NCVS) * 128;
                uint8_t* et = sm + OFF_E + c * 2 * TILE + hf * TILE;  // this warp's 64 columns
#pragma unroll 1
                for (int q2 = 0; q2 < 2; ++q2) {
                    const int jc = 64 * hf + 32 * q2;  // first column of the group within the chunk
                    uint32_t u[32];
                    tc::tc_fence_after();
                    tc::tmem_ld32(tS + 128 * b + lanebase + jc, u);
                    tc::tmem_wait_ld();
                    if (q2 == 1) {  // every score of the chunk this warp needs is in registers
                        tc::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(bar + B_SEMPTY + b);
                    }
                    const int cg = r0 - W + 128 * c + jc;
                    const bool all_in = (cg >= rw0 + 31 - W) && (cg + 31 <= rw0 + W);
                    const bool all_out = (cg + 31 < rw0 - W) || (cg > rw0 + 31 + W);
                    uint32_t ep[16];
                    if (all_out) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) ep[j] = 0u;
                    } else if (all_in) {
                        group_exp<false>(u, cvc + jc, c2, rd2, r - cg, W, ep, acc4);
                    } else {
                        group_exp<true>(u, cvc + jc, c2, rd2, r - cg, W, ep, acc4);
                    }
                    // the previous tile's column sums must have read E chunk c
                    if (q2 == 0 && it >= 1 && !ctl.wait(B_CS + c, (it - 1) & 1)) { ok = false; break; }
                    // E of these 32 columns: 16-byte chunks 4 q2 + q of the half tile
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4*>(et + tc::sw128_off(lr, 4 * q2 + q)) =
                            make_uint4(ep[4 * q], ep[4 * q + 1], ep[4 * q + 2], ep[4 * q + 3]);
                }
                if (!ok) break;
                // the previous tile's column sums of chunk c (complete: waited above)
                if (it >= 1 && hf == 0) {
                    tc::tc_fence_after();
                    put_partial(it - 1, pbh, prb, c);
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar + B_CVEMPTY + (it & 1));
            // ------------------------------------------------ end of tile
            // Parts 1-3 of a quadrant hand their partial row sums to part 0 and go
            // on to the next tile; part 0 forms u, 1/r and the quadrant's scale.
            tc::fence_async_smem();  // this warp's E stores, for the column MMAs
            float* rq = red + (it & 1) * 512 + qd * 128;
            float a0, a1, a2, a3;
            tc::upk2(acc4[0], a0, a1);
            tc::upk2(acc4[1], a2, a3);
            const float rpart = (a0 + a1) + (a2 + a3);
            if (pt != 0) {
                // part 0 has read this buffer's previous contents (and arrived on
                // WFULL for the previous tile) once it released tile it - 1
                if (it >= 1 && !ctl.wait(B_QE + qd, (it - 1) & 1)) { ok = false; break; }
                rq[(pt - 1) * 32 + lane] = rpart;
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    tc::mbar_arrive(bar + B_QF + qd);
                    tc::mbar_arrive(bar + B_WFULL);
                }
            } else {
                if (!ctl.wait(B_QF + qd, it & 1)) { ok = false; break; }
                const float rs = rpart + ((rq[lane] + rq[32 + lane]) + rq[64 + lane]);
                const float w = (rok && rs > 0.f) ? 1.f / rs : 0.f;  // rs > 0 on valid rows
                float wm = w;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
                if (r < L) a.u_out.at(bh, r) = rok ? (rd2 - lg2(rs)) * kLn2 : 0.f;
                // elements (2qd, i) and (2qd + 1, i) of the K-major 16 x 128 operand
                // (two 64-wide K blocks)
                const float wn = wm > 0.f ? w / wm : 0.f;
                const __half hi = __float2half_rn(wn);
                const __half lo = __float2half_rn(wn - __half2float(hi));
                const int kb = lr >> 6, ii = lr & 63, n0 = 2 * qd, n1 = 2 * qd + 1;
                uint8_t* wb = sm + OFF_W + kb * 2048 + 2 * (ii & 7);
                *reinterpret_cast<__half*>(wb + n0 * 128 + ((((ii >> 3) ^ n0) & 7) << 4)) = hi;
                *reinterpret_cast<__half*>(wb + n1 * 128 + ((((ii >> 3) ^ n1) & 7) << 4)) = lo;
                if (lane == 0) wmring[(it % NWM) * 4 + qd] = wm;
                tc::fence_async_smem();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    tc::mbar_arrive(bar + B_WFULL);
                    tc::mbar_arrive(bar + B_QE + qd);
                }
            }
        }
        // the last tile's partials
        if (ok && ntl >= 1 && !*abort_flag && ctl.wait(B_CS + nch - 1, (ntl - 1) & 1)) {
            tc::tc_fence_after();
            for (int c = pt; c < nch; c += NQ) put_partial(ntl - 1, bh, rb, c);
            tc::tc_fence_before();
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, 512);
    }
}

// v_k = v_{k-1} - log(sum of the partials of the row blocks covering each column),
// zero on masked columns.
__global__ void k_finalize_v(const FusedArgs a, MVec v_final) {
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= (long long)a.BH * a.L) return;
    const int bh = (int)(g / a.L), col = (int)(g % a.L);
    const uint8_t* mk_ = a.mask ? a.mask + (size_t)(bh / a.H) * a.L : nullptr;
    const bool valid = !mk_ || mk_[col];
    v_final.at(bh, col) = valid ? v_from_partials(a, bh, col) : 0.f;
}

}  // namespace tcf
}  // namespace sa
