// SIMT band sweeps: every step of the forward and backward as one kernel
// template over (row block x column chunk) tiles of the band.
//
// A "sweep" walks the band row by row.  Rows are the tokens of one side
// (queries for a u-update, keys for a v-update: the band and the mask are
// symmetric, so a column sweep is a row sweep of the transposed problem with
// Q and K, and u and v, exchanged).  For a block of BM rows the columns in
// [r0 - W, r0 + BM - 1 + W] are visited in chunks of BN; each chunk recomputes
// its score tile s = <A_r, B_c> in fp32 FFMA from the stored operands (nothing
// of size L*W is kept), then applies one of the epilogues:
//
//   LSE  : out_r = -log sum_c exp(c*s + e_c)                 (a dual update)
//   WSUM : out_r = base_r + sgn*mult_r * sum_c exp(c*s + d_r + e_c) w_c
//   PV   : out_r = sum_c exp(c*s + d_r + e_c) X_c  (and optionally <Y_r, out_r>)
//   DS1  : out_r = c * sum_c P_rc M_rc X_c,  P = exp(c*s + d_r + e_c),
//          M = G + sum_k rv_k[r] cv_k[c],  G = <A2_r, B2_c>     (one reference)
//   DSD  : out_r = c * sum_c [sum_k exp(c*s + er_k[r] + ec_k[c]) (g_k G + cr_k[r] + cc_k[c])] X_c
//                                                              (direct schedule)
//
// With a dustbin the column side carries one more column (index L) with the
// constant score sd; an extra CTA per problem computes the dustbin ROW of the
// sweep, which touches every token (an O(L) reduction).
//
// Exponentials are evaluated in base 2 (scores and duals scaled by log2 e).
#pragma once

#include "common.cuh"

namespace sa {
namespace simt {

constexpr int D = 64;     // head dimension handled by these kernels
constexpr int BM = 64;    // rows per block
constexpr int BN = 64;    // columns per chunk
constexpr int NT = 256;   // threads per block: 16 x 16, each owning 4 x 4 entries
constexpr int LDT = 68;   // leading dimension (floats) of [D][LDT] transposed tiles
constexpr int LDX = 68;   // leading dimension of [64][LDX] row-major tiles
constexpr int MAXT = 8;   // modifier / staircase terms (2R for R <= 4)

enum Mode { LSE = 0, WSUM = 1, PV = 2, DS1 = 3, DSD = 4 };

struct SweepArgs {
    int L, W, H, ld;        // length, band, heads, dual leading length (L + dustbin)
    float c2;               // score scale * log2(e)
    int dustbin;            // 1: add the dustbin column (and the dustbin-row CTA if dust_cta)
    int dust_cta;           // 1: launch computes the dustbin row in an extra CTA
    float sd2;              // dustbin score * log2(e)
    const void* A;          // row-side score operand [BH][L][D]
    const void* Bo;         // column-side score operand [BH][L][D]
    const void* A2;         // DS: row-side operand of G
    const void* B2;         // DS: column-side operand of G
    const void* X;          // PV/DS: column-side value operand
    const void* Y;          // PV: row-side operand of the dot <Y_r, out_r> (or null)
    const float* Xd;        // PV: dustbin column's value [H][D] (or null = 0)
    const float* Yd;        // PV dustbin row: operand of the dot [H][D] (or null)
    const uint8_t* mask;    // [B][L] (or null)
    Vec rd;                 // row-side dual in the exponent (natural units)
    Vec cd;                 // column-side dual in the exponent
    Vec w;                  // WSUM weights (column side)
    Vec base;               // WSUM additive term (row side; p null = 0)
    Vec mult;               // WSUM multiplier (row side; p null = 1)
    float sgn;              // WSUM sign
    MVec out_vec;           // LSE/WSUM/PV-dot output (row side)
    void* out_mat;          // PV/DS output [BH][L][D]
    float out_scale;        // DS: natural score scale c
    int nterms;             // DS1: rank terms; DSD: staircase terms
    Vec rv[MAXT], cv[MAXT];                  // DS1 (p null = 1)
    Vec er[MAXT], ec[MAXT], cr[MAXT], cc[MAXT];  // DSD (cr/cc p null = 0)
    float gk[MAXT];                          // DSD: weight of G in term k
    float* dvd_part;        // PV dustbin row: [BH][D] sum_c P_(dust,c) X_c (or null)
    // DS with more than MAXT terms runs one launch per block of terms; the
    // launches sum their results in fp32 (plain read-add-write: every output row
    // has one writer per launch and launches are stream ordered)
    float* acc;             // fp32 running sum [BH][L][D]
    int acc_in;             // 1: add acc's contents to this launch's result
    int acc_out;            // 1: write the sum to acc instead of out_mat
    int g_off;              // DS1: leave G out of M (every block but the first)
    // DS1 on tensor cores with at most five terms: the modifier's K16 operands,
    // bf16 [BH][L][16], row side (hi, hi, lo) and column side (hi, lo, hi) of each
    // term (or null: the modifier is formed in the epilogue)
    const void* aug_row;
    const void* aug_col;
    int online;             // LSE on tensor cores: 1 = no previous dual, use a running max
    // Row-sum sweeps on tensor cores (shifted LSE, WSUM): the duals as working
    // copies, log2(e) times the dual on valid tokens and -inf on masked ones
    // ([BH][L], stride s), which the loader copies to shared memory as they are
    int* status;            // the workspace's status word (debug bounds checks)
    Vec cdw;                // column side
    Vec rdw;                // row side (LSE: the shift source; WSUM: the row dual)
    MVec outw;              // LSE: the new dual's working copy (or p null)
    // and the column side's dual as a score-MMA operand row, bf16 [BH][..][L][16]
    // (element (bh, t) at augc + bh * aug_s + 16 t), and the LSE output's row
    const void* augc;
    void* augo;
    long long aug_s;
};

// ---------------------------------------------------------------------------
// tile loads: 64 tokens x 64 dims, zero outside [0, L)
// ---------------------------------------------------------------------------
template <typename T, bool TRANS>
__device__ __forceinline__ void load_tile(float* sm, const T* base, int t0, int L) {
    constexpr int VW = VecW<T>::n;           // elements per 16-byte load
    constexpr int PER_TOK = D / VW;
    for (int idx = threadIdx.x; idx < 64 * PER_TOK; idx += NT) {
        const int tok = idx / PER_TOK;
        const int k0 = (idx % PER_TOK) * VW;
        const int t = t0 + tok;
        float v[8];
        if (t >= 0 && t < L) {
            load_vec(base + (size_t)t * D + k0, v, VW);
        } else {
#pragma unroll
            for (int e = 0; e < VW; ++e) v[e] = 0.f;
        }
        if (TRANS) {
#pragma unroll
            for (int e = 0; e < VW; ++e) sm[(k0 + e) * LDT + tok] = v[e];
        } else {
#pragma unroll
            for (int e = 0; e < VW; e += 4)
                *reinterpret_cast<float4*>(&sm[tok * LDX + k0 + e]) =
                    make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
    }
}

// acc[i][j] = sum_k As[k][ty*4+i] * Bs[k][tx*4+j]
__device__ __forceinline__ void tile_gemm(const float* As, const float* Bs, float acc[4][4],
                                          int ty, int tx) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
    for (int k = 0; k < D; ++k) {
        const float4 a = *reinterpret_cast<const float4*>(&As[k * LDT + ty * 4]);
        const float4 b = *reinterpret_cast<const float4*>(&Bs[k * LDT + tx * 4]);
        const float av[4] = {a.x, a.y, a.z, a.w};
        const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
}

// oacc[i][j] += sum_c Ps[ty*4+i][c] * Xs[c][tx*4+j]
__device__ __forceinline__ void pv_gemm(const float* Ps, const float* Xs, float oacc[4][4],
                                        int ty, int tx) {
#pragma unroll 4
    for (int c = 0; c < BN; ++c) {
        const float4 x = *reinterpret_cast<const float4*>(&Xs[c * LDX + tx * 4]);
        const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float p = Ps[(ty * 4 + i) * LDX + c];
#pragma unroll
            for (int j = 0; j < 4; ++j) oacc[i][j] = fmaf(p, xv[j], oacc[i][j]);
        }
    }
}

__host__ __device__ constexpr int smem_floats(int mode) {
    // As, Bs always; A2s, B2s for DS; Xs, Ps for PV/DS; column vectors
    return (2 + ((mode == DS1 || mode == DSD) ? 2 : 0) + ((mode >= PV) ? 2 : 0)) * (64 * LDT) +
           4 * BN + 2 * MAXT * BN;
}

// ---------------------------------------------------------------------------
// the dustbin row of a sweep (one CTA per problem)
// ---------------------------------------------------------------------------
template <typename T, int MODE>
__device__ void dustbin_row(const SweepArgs& a, int bh, float* sm) {
    const int L = a.L, tid = threadIdx.x;
    const uint8_t* mk = a.mask ? a.mask + (size_t)(bh / a.H) * L : nullptr;
    const float ce_d = a.cd.at(bh, L) * kLog2e;
    const float rd_d = (MODE == LSE) ? 0.f : a.rd.at(bh, L) * kLog2e;
    if (MODE == LSE) {
        float m = -INFINITY, s = 0.f;
        for (int c = tid; c < L; c += NT) {
            if (mk && !mk[c]) continue;
            lse_merge(m, s, a.sd2 + a.cd.at(bh, c) * kLog2e, 1.f);
        }
        if (tid == 0) lse_merge(m, s, a.sd2 + ce_d, 1.f);
        float* ms = sm;
        float* ss = sm + NT;
        ms[tid] = m;
        ss[tid] = s;
        __syncthreads();
        for (int off = NT / 2; off > 0; off >>= 1) {
            if (tid < off) {
                float m1 = ms[tid], s1 = ss[tid];
                lse_merge(m1, s1, ms[tid + off], ss[tid + off]);
                ms[tid] = m1;
                ss[tid] = s1;
            }
            __syncthreads();
        }
        if (tid == 0) a.out_vec.at(bh, L) = -(ms[0] + lg2(ss[0])) * kLn2;
    } else if (MODE == WSUM) {
        float s = 0.f;
        for (int c = tid; c < L; c += NT) {
            if (mk && !mk[c]) continue;
            s += ex2(a.sd2 + rd_d + a.cd.at(bh, c) * kLog2e) * a.w.at(bh, c);
        }
        if (tid == 0) s += ex2(a.sd2 + rd_d + ce_d) * a.w.at(bh, L);
        sm[tid] = s;
        __syncthreads();
        for (int off = NT / 2; off > 0; off >>= 1) {
            if (tid < off) sm[tid] += sm[tid + off];
            __syncthreads();
        }
        if (tid == 0) {
            const float b = a.base.p ? a.base.at(bh, L) : 0.f;
            const float m = a.mult.p ? a.mult.at(bh, L) : 1.f;
            a.out_vec.at(bh, L) = b + a.sgn * m * sm[0];
        }
    } else if (MODE == PV) {
        // dustbin row of the transposed (key-side) sweep: sum_c P_(dust,c) X_c
        const T* Xb = (const T*)a.X + (size_t)bh * L * D;
        const int e = tid % D, part = tid / D;  // 4 partial sums per column
        float s = 0.f;
        for (int c = part; c < L; c += NT / D) {
            if (mk && !mk[c]) continue;
            const float p = ex2(a.sd2 + rd_d + a.cd.at(bh, c) * kLog2e);
            s = fmaf(p, to_f32(Xb[(size_t)c * D + e]), s);
        }
        sm[tid] = s;
        __syncthreads();
        if (tid < D) {
            float v = sm[tid] + sm[tid + D] + sm[tid + 2 * D] + sm[tid + 3 * D];
            if (a.dvd_part) a.dvd_part[(size_t)bh * D + tid] = v;
            sm[4 * D + tid] = (a.Yd ? a.Yd[(size_t)(bh % a.H) * D + tid] : 0.f) * v;
        }
        __syncthreads();
        if (tid == 0 && a.out_vec.p) {
            float dot = 0.f;
            for (int t = 0; t < D; ++t) dot += sm[4 * D + t];
            a.out_vec.at(bh, L) = dot;
        }
    }
}

// ---------------------------------------------------------------------------
// the sweep kernel
// ---------------------------------------------------------------------------
template <typename T, int MODE>
__global__ void __launch_bounds__(NT) band_sweep(const SweepArgs a) {
    extern __shared__ __align__(16) float sm[];
    const int bh = blockIdx.y;
    const int L = a.L, W = a.W;
    const int nblk = (L + BM - 1) / BM;
    if ((int)blockIdx.x >= nblk) {
        if (MODE != DS1 && MODE != DSD) dustbin_row<T, MODE>(a, bh, sm);
        return;
    }
    constexpr bool DS = (MODE == DS1 || MODE == DSD);
    constexpr bool HASX = (MODE == PV || DS);
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int r0 = blockIdx.x * BM;
    const uint8_t* mk = a.mask ? a.mask + (size_t)(bh / a.H) * L : nullptr;
    const size_t off = (size_t)bh * L * D;

    float* As = sm;
    float* Bs = As + 64 * LDT;
    float* A2s = Bs + 64 * LDT;
    float* B2s = DS ? A2s + 64 * LDT : A2s;
    float* Xs = DS ? B2s + 64 * LDT : A2s;
    float* Ps = Xs + 64 * LDT;
    float* colv = HASX ? Ps + 64 * LDT : Xs;   // [4][BN]: exponent dual, weight, valid
    float* ce = colv;
    float* cw = colv + BN;
    float* cvalid = colv + 2 * BN;
    float* cmod = colv + 4 * BN;                // [2*MAXT][BN]

    load_tile<T, true>(As, (const T*)a.A + off, r0, L);
    if (DS) load_tile<T, true>(A2s, (const T*)a.A2 + off, r0, L);

    // row-side values of this thread's 4 rows
    int rr[4];
    bool rv_ok[4];
    float rd2[4];
    float rmod[MAXT][4];    // DS1: rv_k; DSD: er_k (base 2)
    float rmod2[MAXT][4];   // DSD: cr_k
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + ty * 4 + i;
        rr[i] = r;
        rv_ok[i] = (r < L) && (mk == nullptr || mk[r] != 0);
        rd2[i] = (MODE != LSE && r < L) ? a.rd.at(bh, r) * kLog2e : 0.f;
#pragma unroll
        for (int k = 0; k < MAXT; ++k) {
            rmod[k][i] = 0.f;
            rmod2[k][i] = 0.f;
            if (k < a.nterms && r < L) {
                if (MODE == DS1) rmod[k][i] = a.rv[k].p ? a.rv[k].at(bh, r) : 1.f;
                if (MODE == DSD) {
                    rmod[k][i] = a.er[k].at(bh, r) * kLog2e;
                    rmod2[k][i] = a.cr[k].p ? a.cr[k].at(bh, r) : 0.f;
                }
            }
        }
    }

    float m[4], s[4];        // LSE: running base-2 max and sum; WSUM: s = sum
    float oacc[4][4];        // PV/DS accumulators (rows x d-columns tx*4+j)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[i] = -INFINITY;
        s[i] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) oacc[i][j] = 0.f;
    }

    const int cbeg = max(0, r0 - W);
    const int cend = min(L, r0 + BM - 1 + W + 1);
    for (int c0 = cbeg; c0 < cend; c0 += BN) {
        __syncthreads();
        load_tile<T, true>(Bs, (const T*)a.Bo + off, c0, L);
        if (DS) load_tile<T, true>(B2s, (const T*)a.B2 + off, c0, L);
        if (HASX) load_tile<T, false>(Xs, (const T*)a.X + off, c0, L);
        if (tid < BN) {
            const int c = c0 + tid;
            const bool ok = (c < cend) && (mk == nullptr || mk[c] != 0);
            cvalid[tid] = ok ? 1.f : 0.f;
            ce[tid] = ok ? a.cd.at(bh, c) * kLog2e : 0.f;
            if (MODE == WSUM) cw[tid] = ok ? a.w.at(bh, c) : 0.f;
            for (int k = 0; k < a.nterms; ++k) {
                if (MODE == DS1) cmod[k * BN + tid] = (ok && a.cv[k].p) ? a.cv[k].at(bh, c) : (ok ? 1.f : 0.f);
                if (MODE == DSD) {
                    cmod[k * BN + tid] = ok ? a.ec[k].at(bh, c) * kLog2e : 0.f;
                    cmod[(MAXT + k) * BN + tid] = (ok && a.cc[k].p) ? a.cc[k].at(bh, c) : 0.f;
                }
            }
        }
        __syncthreads();

        float acc[4][4];
        tile_gemm(As, Bs, acc, ty, tx);
        float g[4][4];
        if (DS) tile_gemm(A2s, B2s, g, ty, tx);

        // support of this thread's 4 x 4 entries
        bool in[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + tx * 4 + j;
                const int dist = rr[i] - c;
                in[i][j] = rv_ok[i] && cvalid[tx * 4 + j] != 0.f && dist <= W && dist >= -W;
            }

        if (MODE == LSE) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float x[4];
                float mloc = -INFINITY;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    x[j] = in[i][j] ? fmaf(a.c2, acc[i][j], ce[tx * 4 + j]) : -INFINITY;
                    mloc = fmaxf(mloc, x[j]);
                }
                if (mloc > m[i]) {
                    s[i] *= ex2(m[i] - mloc);
                    m[i] = mloc;
                }
                if (m[i] != -INFINITY) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) s[i] += ex2(x[j] - m[i]);
                }
            }
        } else if (MODE == WSUM) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (in[i][j])
                        s[i] = fmaf(ex2(fmaf(a.c2, acc[i][j], rd2[i] + ce[tx * 4 + j])),
                                    cw[tx * 4 + j], s[i]);
        } else {
            // P (PV) or dS (DS) into Ps, then accumulate Ps x Xs
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float pr[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float val = 0.f;
                    if (in[i][j]) {
                        const int cj = tx * 4 + j;
                        if (MODE == PV) {
                            val = ex2(fmaf(a.c2, acc[i][j], rd2[i] + ce[cj]));
                        } else if (MODE == DS1) {
                            float M = a.g_off ? 0.f : g[i][j];
#pragma unroll
                            for (int k = 0; k < MAXT; ++k)
                                if (k < a.nterms) M = fmaf(rmod[k][i], cmod[k * BN + cj], M);
                            val = ex2(fmaf(a.c2, acc[i][j], rd2[i] + ce[cj])) * M;
                        } else {
#pragma unroll
                            for (int k = 0; k < MAXT; ++k) {
                                if (k < a.nterms) {
                                    const float pk = ex2(fmaf(a.c2, acc[i][j], rmod[k][i] + cmod[k * BN + cj]));
                                    const float coef = a.gk[k] * g[i][j] + rmod2[k][i] +
                                                       cmod[(MAXT + k) * BN + cj];
                                    val = fmaf(pk, coef, val);
                                }
                            }
                        }
                    }
                    pr[j] = val;
                }
                *reinterpret_cast<float4*>(&Ps[(ty * 4 + i) * LDX + tx * 4]) =
                    make_float4(pr[0], pr[1], pr[2], pr[3]);
            }
            __syncthreads();
            pv_gemm(Ps, Xs, oacc, ty, tx);
        }
    }

    // ---- finish: dustbin column, reduction over the 16 lanes of a row, store
    const float ce_d = a.dustbin ? a.cd.at(bh, L) * kLog2e : 0.f;
    if (MODE == LSE) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (a.dustbin && tx == 0 && rv_ok[i]) lse_merge(m[i], s[i], a.sd2 + ce_d, 1.f);
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, m[i], o);
                const float s2 = __shfl_xor_sync(0xffffffffu, s[i], o);
                lse_merge(m[i], s[i], m2, s2);
            }
            if (tx == 0 && rr[i] < L && SA_BOUNDS(rr[i] >= 0 && bh < (int)gridDim.y, a.status))
                a.out_vec.at(bh, rr[i]) = rv_ok[i] ? -(m[i] + lg2(s[i])) * kLn2 : 0.f;
        }
    } else if (MODE == WSUM) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (a.dustbin && tx == 0 && rv_ok[i]) s[i] += ex2(a.sd2 + rd2[i] + ce_d) * a.w.at(bh, L);
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) s[i] += __shfl_xor_sync(0xffffffffu, s[i], o);
            if (tx == 0 && rr[i] < L && SA_BOUNDS(rr[i] >= 0 && bh < (int)gridDim.y, a.status)) {
                float v = 0.f;
                if (rv_ok[i]) {
                    const float b = a.base.p ? a.base.at(bh, rr[i]) : 0.f;
                    const float mu = a.mult.p ? a.mult.at(bh, rr[i]) : 1.f;
                    v = b + a.sgn * mu * s[i];
                }
                a.out_vec.at(bh, rr[i]) = v;
            }
        }
    } else {
        if (MODE == PV && a.dustbin && a.Xd) {
            const float* xd = a.Xd + (size_t)(bh % a.H) * D + tx * 4;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (!rv_ok[i]) continue;
                const float p = ex2(a.sd2 + rd2[i] + ce_d);
#pragma unroll
                for (int j = 0; j < 4; ++j) oacc[i][j] = fmaf(p, xd[j], oacc[i][j]);
            }
        }
        const float scale = DS ? a.out_scale : 1.f;
        T* outb = (T*)a.out_mat + off;
        const T* Yb = (MODE == PV && a.Y) ? (const T*)a.Y + off : nullptr;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = rr[i];
            float dot = 0.f;
            float o4[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) o4[j] = rv_ok[i] ? oacc[i][j] * scale : 0.f;
            if (r < L && SA_BOUNDS(r >= 0 && bh < (int)gridDim.y && tx * 4 + 4 <= D, a.status)) {
                float* accr = (DS && a.acc) ? a.acc + off + (size_t)r * D + tx * 4 : nullptr;
                if (DS && accr && a.acc_in) {
                    const float4 p = *reinterpret_cast<const float4*>(accr);
                    o4[0] += p.x; o4[1] += p.y; o4[2] += p.z; o4[3] += p.w;
                }
                if (DS && accr && a.acc_out)
                    *reinterpret_cast<float4*>(accr) = make_float4(o4[0], o4[1], o4[2], o4[3]);
                else
                    store4(outb + (size_t)r * D + tx * 4, o4[0], o4[1], o4[2], o4[3]);
                if (Yb) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) dot = fmaf(to_f32(Yb[(size_t)r * D + tx * 4 + j]), o4[j], dot);
                }
            }
            if (Yb) {
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                if (tx == 0 && r < L && a.out_vec.p) a.out_vec.at(bh, r) = rv_ok[i] ? dot : 0.f;
            }
        }
    }
}

}  // namespace simt
}  // namespace sa
