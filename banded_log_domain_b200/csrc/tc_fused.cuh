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
// known the MMA computes D[j, n] = sum_i E[i, j] w[i, n] with w = 1/r split
// into fp16 high and low parts (columns n = 0, 1), scaled by the block's
// largest 1/r.
//
// Persistent CTAs (one per SM) walk the (batch*head, row block) tiles.  Warp
// roles: warps 0-15 epilogue (TMEM lane quadrant w%4, 32-column quarter w/4 of
// each chunk), warp 16 TMA loader (Q blocks, K chunks), warp 17 MMA issuer
// (score tiles, and the previous tile's column sums after the next tile's first
// two score tiles), warps 18-19 the next tile's column duals.  Every mbarrier
// wait is bounded.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace sa {
namespace tcf {

constexpr int NEPI = 16;           // epilogue warps: lane quadrant (w % 4) x column part (w / 4)
constexpr int NQ = NEPI / 4;       // column parts per 128-column chunk
constexpr int PW = 128 / NQ;       // columns per part
constexpr int GP = PW / 32;        // 32-column groups per part
constexpr int W_LOAD = NEPI, W_MMA = NEPI + 1, W_CV = NEPI + 2;  // two column-dual warps
constexpr int NTHREADS = (NEPI + 4) * 32;
constexpr int NSLOT = 8;          // partial slots per column
constexpr int TILE = 16384;        // 128 x 64 bf16 (or 128 x 64 fp16) swizzled tile
constexpr int NST = 2;             // K-chunk stages
constexpr int MAXCH = 5;           // column chunks per row block (2W + 128 <= 640)
constexpr int MAXCOL = 128 * MAXCH;
constexpr long long kWaitBudget = 4000000000LL;

// shared-memory carve-up (from a 1024-aligned base)
constexpr int OFF_A = 0;
constexpr int OFF_STAGE = TILE;
constexpr int OFF_E = OFF_STAGE + NST * TILE;
constexpr int OFF_W = OFF_E + MAXCH * 2 * TILE;  // 16 x 128 fp16, two 2 KB K-blocks
constexpr int OFF_CV = OFF_W + 4096;             // 2 x MAXCOL floats
constexpr int OFF_RED = OFF_CV + 2 * MAXCOL * 4; // NQ x 128 floats, then 4 floats
constexpr int OFF_BAR = OFF_RED + 4 * 128 * 4 + 64;
constexpr int SMEM_BYTES = OFF_BAR + 32 * 8 + 16 + 1024;

enum { B_AFULL = 0, B_AEMPTY = 1, B_FULL = 2, B_EMPTY = 4, B_SFULL = 6, B_SEMPTY = 8,
       B_CVFULL = 10, B_CVEMPTY = 12, B_WFULL = 14, B_DRAIN = 15, B_EPI = 16,
       B_CS = 17 /* .. 17 + MAXCH - 1: column sums of chunk c done */ };

struct FusedArgs {
    int L, W, H, BH, nblk, ncol, nch;  // ncol = 2W + 128, nch = ceil(ncol / 128)
    float c2;                          // score scale * log2(e)
    const uint8_t* mask;               // [B][L] or null
    Vec u_prev;                        // u_{k-1}
    MVec u_out;                        // u_k (may alias u_prev)
    Vec v_src;                         // v_{k-1} (materialised) or v_{k-2} (with part_in)
    MVec v_out;                        // with part_in: v_{k-1} of the owned columns
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

__device__ __forceinline__ void tmem_ld2(uint32_t taddr, uint32_t& r0, uint32_t& r1) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(taddr)
                 : "memory");
}

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

// v_{k-1} of column `col` from v_{k-2} and the covering row blocks' partials.
__device__ __forceinline__ float v_from_partials(const FusedArgs& a, int bh, int col) {
    const int x = col - 127 - a.W;
    const int lo = x <= 0 ? 0 : (x + 127) / 128;
    const int hi = min(a.nblk - 1, (col + a.W) / 128);
    const float4* p = reinterpret_cast<const float4*>(a.part_in + ((size_t)bh * a.L + col) * NSLOT);
    const float4 p0 = p[0], p1 = p[1];
    const float sl[NSLOT] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < NSLOT; ++i) {  // row block lo + i, slot (lo + i) mod 8
        if (lo + i <= hi) sum += sl[(lo + i) & (NSLOT - 1)];
    }
    return a.v_src.at(bh, col) - lg2(sum) * kLn2;
}

// E = exp2(c2 * s + cv + rd2) for one thread's 32 columns; `CHECK` masks the
// entries off the band (only the groups that straddle the band's edge).
template <bool CHECK>
__device__ __forceinline__ void group_exp(const uint32_t (&u)[32], const float* cvp, float c2,
                                          float rd2, int d_first, int W, float (&e)[32],
                                          float (&acc4)[4]) {
    const float4* c4 = reinterpret_cast<const float4*>(cvp);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 cvv = c4[q];
        float x0 = fmaf(__uint_as_float(u[4 * q]), c2, cvv.x + rd2);
        float x1 = fmaf(__uint_as_float(u[4 * q + 1]), c2, cvv.y + rd2);
        float x2 = fmaf(__uint_as_float(u[4 * q + 2]), c2, cvv.z + rd2);
        float x3 = fmaf(__uint_as_float(u[4 * q + 3]), c2, cvv.w + rd2);
        if (CHECK) {
            const int d0 = d_first - 4 * q;  // row - column of element 4q
            if ((unsigned)(d0 + W) > (unsigned)(2 * W)) x0 = -INFINITY;
            if ((unsigned)(d0 - 1 + W) > (unsigned)(2 * W)) x1 = -INFINITY;
            if ((unsigned)(d0 - 2 + W) > (unsigned)(2 * W)) x2 = -INFINITY;
            if ((unsigned)(d0 - 3 + W) > (unsigned)(2 * W)) x3 = -INFINITY;
        }
        e[4 * q] = ex2(x0);
        e[4 * q + 1] = ex2(x1);
        e[4 * q + 2] = ex2(x2);
        e[4 * q + 3] = ex2(x3);
        acc4[0] += e[4 * q];
        acc4[1] += e[4 * q + 1];
        acc4[2] += e[4 * q + 2];
        acc4[3] += e[4 * q + 3];
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
    float* cvbuf = reinterpret_cast<float*>(sm + OFF_CV);
    float* red = reinterpret_cast<float*>(sm + OFF_RED);
    float* red2 = red + 512;
    Ctl ctl{bar, abort_flag, a.status};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = a.BH * a.nblk;
    const int L = a.L, W = a.W, nch = a.nch, ncol = a.ncol;

    // zero the 1/r operand once (rows n >= 2 stay zero)
    for (int t = threadIdx.x; t < 4096 / 16; t += NTHREADS)
        reinterpret_cast<uint4*>(sm + OFF_W)[t] = make_uint4(0, 0, 0, 0);
    tc::fence_async_smem();
    if (threadIdx.x == 0) {
        tc::mbar_init(bar + B_AFULL, 1);
        tc::mbar_init(bar + B_AEMPTY, 1);
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bar + B_FULL + i, 1);
            tc::mbar_init(bar + B_EMPTY + i, 1);
            tc::mbar_init(bar + B_SFULL + i, 1);
            tc::mbar_init(bar + B_SEMPTY + i, NEPI);
            tc::mbar_init(bar + B_CVFULL + i, 64);
            tc::mbar_init(bar + B_CVEMPTY + i, NEPI);
        }
        tc::mbar_init(bar + B_WFULL, NEPI);
        for (int c = 0; c < MAXCH; ++c) tc::mbar_init(bar + B_CS + c, 1);
        tc::mbar_init(bar + B_DRAIN, 1);
        tc::mbar_init(bar + B_EPI, NEPI);
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
    // TMEM: S buffers at columns 0 and 128; column sums at 256 + 32c (+16 for odd K steps)
    const uint32_t tS = tm, tD = tm + 256;

    if (warp == W_CV || warp == W_CV + 1) {
        // ------------------------------------------------------------ column duals
        const int ln = (warp - W_CV) * 32 + lane;  // 0..63
        int it = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
            const int bh = t / a.nblk, rb = t % a.nblk, r0 = rb * 128;
            const uint8_t* mk_ = a.mask ? a.mask + (size_t)(bh / a.H) * L : nullptr;
            const int cb = it & 1;
            if (it >= 2 && !ctl.wait(B_CVEMPTY + cb, ((it >> 1) - 1) & 1)) break;
            float* cv = cvbuf + cb * MAXCOL;
#pragma unroll 4
            for (int cc = ln; cc < nch * 128; cc += 64) {
                const int col = r0 - W + cc;
                const bool valid = cc < ncol && col >= 0 && col < L && (!mk_ || mk_[col]);
                float v = 0.f;
                if (valid) v = a.part_in ? v_from_partials(a, bh, col) : a.v_src.at(bh, col);
                if (a.part_in && a.v_out.p && col >= r0 && col < r0 + 128 && col < L)
                    a.v_out.at(bh, col) = valid ? v : 0.f;
                cv[cc] = valid ? v * kLog2e : -INFINITY;
            }
            tc::mbar_arrive(bar + B_CVFULL + cb);
        }
    } else if (warp == W_LOAD) {
        // ------------------------------------------------------------ TMA loader
        if (lane == 0) {
            int gc = 0, it = 0, issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++it) {
                const int bh = t / a.nblk, rb = t % a.nblk, r0 = rb * 128;
                if (it >= 1 && !ctl.wait(B_AEMPTY, (it - 1) & 1)) break;
                tc::mbar_expect_tx(bar + B_AFULL, TILE);
                tc::tma_load_3d(sm + OFF_A, &mq, bar + B_AFULL, 0, r0, bh);
                for (int c = 0; ok && c < nch; ++c, ++gc) {
                    const int s = gc % NST;
                    if (gc >= NST && !ctl.wait(B_EMPTY + s, ((gc / NST) - 1) & 1)) { ok = false; break; }
                    tc::mbar_expect_tx(bar + B_FULL + s, TILE);
                    tc::tma_load_3d(sm + OFF_STAGE + s * TILE, &mk, bar + B_FULL + s, 0,
                                    r0 - W + 128 * c, bh);
                    issued = gc + 1;
                }
            }
            if (*abort_flag) {  // let issued loads land before teardown
                for (int g = max(0, issued - NST); g < issued; ++g)
                    tc::mbar_wait(bar + B_FULL + g % NST, (g / NST) & 1, kWaitBudget);
            }
        }
        __syncwarp();
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = tc::idesc_bf16(128, 128, false, false);
            const uint32_t id_c = idesc_f16(128, 16, true, false);
            // descriptors built once; offsets are added in 16-byte units
            const uint64_t dA = tc::sdesc_sw128(tc::smem_u32(sm + OFF_A), 16, 1024);
            const uint64_t dSt = tc::sdesc_sw128(tc::smem_u32(sm + OFF_STAGE), 16, 1024);
            const uint64_t dE = tc::sdesc_sw128(tc::smem_u32(sm + OFF_E), TILE, 1024);
            uint64_t dW[8];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                dW[kk] = tc::sdesc_sw128(tc::smem_u32(sm + OFF_W) + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);
            bool ok = true;
            // column sums of tile t_it: D[j, n] = sum_i E[i, j] w[i, n], two
            // accumulators per chunk (even / odd K steps); chunk c's commit frees
            // its E tile
            auto do_col = [&](int t_it) {
                if (!ctl.wait(B_WFULL, t_it & 1)) { ok = false; return; }
                tc::tc_fence_after();
                for (int c = 0; c < nch; ++c) {
                    const uint64_t dEc = tc::sdesc_add(dE, c * 2 * TILE);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_bf16(tD + 32 * c + 16 * (kk & 1), tc::sdesc_add(dEc, kk * 2048), dW[kk],
                                     id_c, kk > 1 ? 1u : 0u);
                    tc::tc_commit(bar + B_CS + c);
                }
            };
            int gc = 0, it = 0;
            for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++it) {
                if (!ctl.wait(B_AFULL, it & 1)) { ok = false; break; }
                for (int c = 0; c < nch; ++c, ++gc) {
                    const int s = gc % NST, b = gc & 1;
                    if (!ctl.wait(B_FULL + s, (gc / NST) & 1)) { ok = false; break; }
                    if (gc >= 2 && !ctl.wait(B_SEMPTY + b, ((gc >> 1) - 1) & 1)) { ok = false; break; }
                    tc::tc_fence_after();
                    const uint64_t dB = tc::sdesc_add(dSt, s * TILE);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_bf16(tS + 128 * b, tc::sdesc_add(dA, 32 * k), tc::sdesc_add(dB, 32 * k),
                                     id_s, k > 0);
                    tc::tc_commit(bar + B_SFULL + b);
                    tc::tc_commit(bar + B_EMPTY + s);
                    if (it >= 1 && c == min(1, nch - 1)) {
                        do_col(it - 1);
                        if (!ok) break;
                    }
                }
                if (!ok) break;
                tc::tc_commit(bar + B_AEMPTY);
            }
            if (ok && it >= 1) do_col(it - 1);
            tc::tc_commit(bar + B_DRAIN);
            tc::mbar_wait(bar + B_DRAIN, 0, kWaitBudget);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int qd = warp & 3, pt = warp >> 2;
        const int lr = qd * 32 + lane;
        const uint32_t lanebase = (uint32_t)(qd * 32) << 16;
        const float c2 = a.c2;
        int gc = 0, it = 0, done = 0;
        uint32_t eph = 0;
        int prev_bh = 0, prev_rb = 0;
        float prev_wmax = 0.f;
        // column partials of tile t_it (its column sums in TMEM buffer t_it & 1)
        auto store_partials = [&](int t_it, int pbh, int prb, float pwmax) -> bool {
            if (!ctl.wait(B_CS + nch - 1, t_it & 1)) return false;  // every column MMA of the tile
            tc::tc_fence_after();
            float* po = a.part_out + (size_t)pbh * L * NSLOT + (prb & (NSLOT - 1));
            const int pr0 = prb * 128;
            for (int c = pt; c < nch; c += NQ) {
                uint32_t d0, d1, d2, d3;
                tmem_ld2(tD + lanebase + 32 * c, d0, d1);
                tmem_ld2(tD + lanebase + 32 * c + 16, d2, d3);
                tc::tmem_wait_ld();
                const int cc = 128 * c + lr, col = pr0 - W + cc;
                if (cc < ncol && col >= 0 && col < L)
                    po[(size_t)col * NSLOT] = ((__uint_as_float(d0) + __uint_as_float(d2)) +
                                               (__uint_as_float(d1) + __uint_as_float(d3))) * pwmax;
            }
            tc::tc_fence_before();
            return true;
        };
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
            const int bh = t / a.nblk, rb = t % a.nblk, r0 = rb * 128;
            const int r = r0 + lr, rw0 = r0 + qd * 32;
            const uint8_t* mk_ = a.mask ? a.mask + (size_t)(bh / a.H) * L : nullptr;
            const bool rok = r < L && (!mk_ || mk_[r]);
            // rows that are not valid get exp(-inf) = 0 everywhere
            const float rd2 = rok ? a.u_prev.at(bh, r) * kLog2e : -INFINITY;
            const int cb = it & 1;
            if (!ctl.wait(B_CVFULL + cb, (it >> 1) & 1)) break;
            const float* cv = cvbuf + cb * MAXCOL;
            float acc4[4] = {0.f, 0.f, 0.f, 0.f};
            bool ok = true;
            for (int c = 0; c < nch; ++c, ++gc) {
                const int b = gc & 1;
                if (!ctl.wait(B_SFULL + b, (gc >> 1) & 1)) { ok = false; break; }
                tc::tc_fence_after();
                uint32_t u[GP][32];
#pragma unroll
                for (int g = 0; g < GP; ++g) tc::tmem_ld32(tS + 128 * b + lanebase + PW * pt + 32 * g, u[g]);
                tc::tmem_wait_ld();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar + B_SEMPTY + b);
                // the previous tile's column sums of chunk c must have read E chunk c
                if (it >= 1 && !ctl.wait(B_CS + c, (it - 1) & 1)) { ok = false; break; }
#pragma unroll
                for (int g = 0; g < GP; ++g) {
                    const int jc = PW * pt + 32 * g;  // first column of this group within the chunk
                    const int cg = r0 - W + 128 * c + jc;
                    const bool all_in = (cg >= rw0 + 31 - W) && (cg + 31 <= rw0 + W);
                    const bool all_out = (cg + 31 < rw0 - W) || (cg > rw0 + 31 + W);
                    float e[32];
                    if (all_out) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) e[j] = 0.f;
                    } else if (all_in) {
                        group_exp<false>(u[g], cv + 128 * c + jc, c2, rd2, r - cg, W, e, acc4);
                    } else {
                        group_exp<true>(u[g], cv + 128 * c + jc, c2, rd2, r - cg, W, e, acc4);
                    }
                    // E of these 32 columns: half jc / 64, 16-byte chunks (jc % 64) / 8 + q
                    uint8_t* et = sm + OFF_E + c * 2 * TILE + (jc >> 6) * TILE;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 w4;
                        w4.x = pack_f16(e[8 * q + 0], e[8 * q + 1]);
                        w4.y = pack_f16(e[8 * q + 2], e[8 * q + 3]);
                        w4.z = pack_f16(e[8 * q + 4], e[8 * q + 5]);
                        w4.w = pack_f16(e[8 * q + 6], e[8 * q + 7]);
                        *reinterpret_cast<uint4*>(et + tc::sw128_off(lr, ((jc & 63) >> 3) + q)) = w4;
                    }
                }
            }
            if (!ok) break;
            // ------------------------------------------------ previous tile's partials
            if (it >= 1 && !store_partials(it - 1, prev_bh, prev_rb, prev_wmax)) break;
            // ------------------------------------------------ end of tile
            tc::fence_async_smem();
            red[pt * 128 + lr] = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
            if (!ctl.epi_sync(eph)) break;
            float w = 0.f;
            if (pt == 0) {
                float rs = 0.f;
#pragma unroll
                for (int k = 0; k < NQ; ++k) rs += red[k * 128 + lr];
                if (r < L) a.u_out.at(bh, r) = rok ? (rd2 - lg2(rs)) * kLn2 : 0.f;  // rs > 0 on valid rows
                w = (rok && rs > 0.f) ? 1.f / rs : 0.f;
                float wm = w;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
                if (lane == 0) red2[qd] = wm;
            }
            if (!ctl.epi_sync(eph)) break;
            const float wmax = fmaxf(fmaxf(red2[0], red2[1]), fmaxf(red2[2], red2[3]));
            if (pt == 0) {
                const float wn = wmax > 0.f ? w / wmax : 0.f;
                const __half hi = __float2half_rn(wn);
                const __half lo = __float2half_rn(wn - __half2float(hi));
                // element (n, i) of the K-major 16 x 128 operand, two 64-wide K blocks
                const int kb = lr >> 6, ii = lr & 63;
                uint8_t* wb = sm + OFF_W + kb * 2048;
                *reinterpret_cast<__half*>(wb + 0 * 128 + ((((ii >> 3) ^ 0) & 7) << 4) + 2 * (ii & 7)) = hi;
                *reinterpret_cast<__half*>(wb + 1 * 128 + ((((ii >> 3) ^ 1) & 7) << 4) + 2 * (ii & 7)) = lo;
                tc::fence_async_smem();
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(bar + B_CVEMPTY + cb);
                tc::mbar_arrive(bar + B_WFULL);
            }
            prev_bh = bh;
            prev_rb = rb;
            prev_wmax = wmax;
            ++done;
        }
        // the last tile's partials
        if (done >= 1 && !*abort_flag) store_partials(done - 1, prev_bh, prev_rb, prev_wmax);
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
