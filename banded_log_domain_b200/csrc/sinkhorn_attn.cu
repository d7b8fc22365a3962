// C ABI of the banded log-domain Sinkhorn attention library: argument
// validation, workspace layout and the launch sequence of each entry point.
//
// Forward (Block-Wise Differentiable Sinkhorn Attention, technical summary
// section 2.1): v0 = 0; T base iterations and R tail iterations, each a row
// sweep (u from v) followed by a column sweep (v from u); then O = P^(R,R) V.
//
// Backward (section 2.2), the one-reference schedule for general R:
//   a      = rowdot(dO, O)
//   dV     = P^T dO,                      vbar^R = rowdot(V, dV)      [key sweep]
//   ubar^R = a - P vbar^R                                             [query sweep]
//   for r = R..2:
//     vbar^(r-1) = -ev^(r-1) . P^T (eu^r . ubar^r)                    [key sweep]
//     ubar^(r-1) = -eu^(r-1) . P (ev^(r-1) . vbar^(r-1))              [query sweep]
//   dS = P . M,  M = G - vbar^R_j - sum_r eu^r_i ev^(r-1)_j ubar^r_i
//                               - sum_{r<R} eu^r_i ev^r_j vbar^r_j
//   dQ = c dS K [query sweep],  dK = c dS^T Q [key sweep]
// where P = P^(R,R), G_ij = <dO_i, V_j>, eu^a = exp(u^(a) - u^(R)) and
// ev^b = exp(v^(b) - v^(R)) (the transport-orbit factors).  The direct
// schedule runs the same sweeps with every staircase plan P^(r,r-1),
// P^(r,r) formed by its own exponential.
#include <cmath>
#include <algorithm>
#include <vector>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include <type_traits>

#include "../../include/sinkhorn_attn.h"
#include "simt_sweep.cuh"
#include "tc_sweep.cuh"
#include "tc_rowsum.cuh"

namespace sa {
namespace {

constexpr size_t kHeader = 256;   // status word + padding at the start of every workspace
constexpr int kD = simt::D;
constexpr int kMaxR = 256;  // tail length limit (host term lists, workspace)
constexpr int kMaxDevicesHS = 64;  // devices with copy streams for the host-buffer step

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

struct Dims {
    int B, H, L, R, ld, BH;
    bool ok;
};

sa_status check_params(const sa_params* p, Dims* dd) {
    if (!p) return SA_ERR_INVALID_ARG;
    if (p->B < 0 || p->H < 0 || p->L < 0 || p->d <= 0 || p->W < 0 || p->T < 0 || p->R < 0)
        return SA_ERR_INVALID_ARG;
    if (!(p->eps > 0.f) || !std::isfinite(p->eps)) return SA_ERR_INVALID_ARG;
    if (p->dtype != SA_F32 && p->dtype != SA_BF16) return SA_ERR_INVALID_ARG;
    if (p->dustbin != 0 && p->dustbin != 1) return SA_ERR_INVALID_ARG;
    if (p->dustbin && !std::isfinite(p->dustbin_score)) return SA_ERR_INVALID_ARG;
    if (p->bwd != SA_BWD_ONE_REFERENCE && p->bwd != SA_BWD_DIRECT) return SA_ERR_INVALID_ARG;
    if (p->check_finite != 0 && p->check_finite != 1) return SA_ERR_INVALID_ARG;
    if (p->d != kD) return SA_ERR_UNSUPPORTED;
    if (p->R > kMaxR) return SA_ERR_UNSUPPORTED;
    const long long BH = (long long)p->B * p->H;
    if (BH > 65535) return SA_ERR_UNSUPPORTED;
    if ((long long)p->L * kD > (1LL << 40)) return SA_ERR_UNSUPPORTED;
    dd->B = p->B;
    dd->H = p->H;
    dd->L = p->L;
    dd->R = p->R;
    dd->ld = p->L + p->dustbin;
    dd->BH = (int)BH;
    dd->ok = true;
    return SA_OK;
}

bool aligned16(const void* x) { return ((uintptr_t)x & 15u) == 0; }

// Memory the current device's kernels may read and write at full speed: device
// memory of the current device, or managed memory.  Pinned host memory (read
// over PCIe), pageable host memory, and another device's memory (a tensor on
// another GPU, or the wrong device current) are rejected before any launch.
bool on_current_device(const void* x) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, x) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (at.type == cudaMemoryTypeManaged) return true;
    if (at.type != cudaMemoryTypeDevice) return false;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.device == dev;
}
bool device_ok(const void* x) { return x && aligned16(x) && on_current_device(x); }
// A device float that may sit anywhere a float may (4-byte alignment).
bool device_f32_ok(const void* x) { return x && ((uintptr_t)x & 3u) == 0 && on_current_device(x); }
// The byte mask (any alignment; NULL means every token is valid).
bool mask_ok(const void* x) { return !x || on_current_device(x); }

// The row-sum sweeps on the tensor cores (bf16 storage without a dustbin) read
// the duals as a working copy of the state: [BH][2R+2][L] float32, log2(e)
// times each dual on valid tokens and -inf on masked ones; then the same duals
// as score-MMA operands, [BH][2R+2][L][16] bf16: slots 0-2 hold a three-way
// bf16 split of dual / c (c the score scale, so the dual is in the units of
// <q, k>), -1e30 on masked tokens, slots 3-15 zero.
bool uses_work_state(const sa_params* p) { return p->dtype == SA_BF16 && !p->dustbin; }
size_t work_floats_bytes(const Dims& d) { return align_up((size_t)d.BH * (2 * d.R + 2) * d.L * sizeof(float)); }
size_t work_aug_bytes(const Dims& d) { return align_up((size_t)d.BH * (2 * d.R + 2) * d.L * 16 * 2); }
size_t work_state_bytes(const Dims& d) { return work_floats_bytes(d) + work_aug_bytes(d); }

// Forward workspace: the status header, then the working copy of the state
// (tensor-core path only).
struct FwdLayout {
    size_t work, total;
};
FwdLayout fwd_layout(const Dims& d, const sa_params* p) {
    FwdLayout l{kHeader, kHeader};
    if (uses_work_state(p)) l.total += work_state_bytes(d);
    return l;
}

// Backward workspace layout (float32 vectors of BH * ld elements each).
struct BwdLayout {
    size_t a, ubar, vbar, eu, ev, w, rv, cv, dvd, dsc, aug, acc, work, total;
    size_t vec;  // bytes of one [BH][ld] vector, 256-aligned
};
BwdLayout bwd_layout(const Dims& d, const sa_params* p) {
    BwdLayout l;
    l.vec = align_up((size_t)d.BH * d.ld * sizeof(float));
    size_t o = kHeader;
    l.a = o;    o += l.vec;
    l.ubar = o; o += l.vec * (d.R + 1);   // index r = 0..R (0 unused)
    l.vbar = o; o += l.vec * (d.R + 1);
    l.eu = o;   o += l.vec * (d.R + 1);
    l.ev = o;   o += l.vec * (d.R + 1);
    l.w = o;    o += l.vec;
    l.rv = o;   o += l.vec * 2 * d.R;
    l.cv = o;   o += l.vec * 2 * d.R;
    l.dvd = o;  o += align_up((size_t)d.BH * kD * sizeof(float));
    l.dsc = o;  o += align_up((size_t)d.BH * sizeof(double));  // dustbin score, per problem
    l.aug = o;  o += 4 * align_up((size_t)d.BH * d.L * 16 * 2);  // bf16 K16 modifier operands
    l.acc = o;  // fp32 sum of the dS sweeps' term blocks, when 2R > MAXT
    if (2 * d.R > simt::MAXT) o += align_up((size_t)d.BH * d.L * kD * sizeof(float));
    l.work = o;  // the working copy of the state (tensor-core path)
    if (uses_work_state(p)) o += work_state_bytes(d);
    l.total = o;
    return l;
}

// ---------------------------------------------------------------------------
// small elementwise kernels
// ---------------------------------------------------------------------------

// out[bh][t] = <X_t, Y_t> over d for valid tokens, 0 for masked ones and for
// the dustbin slot t = L.  A token's row is read by kD / (16 / sizeof(T)) lanes,
// one 16-byte load per tensor each (coalesced), and summed with shuffles.
template <typename T>
__global__ void k_rowdot(const T* X, const T* Y, const uint8_t* mask, int L, int H, int ld,
                         int BH, float* out) {
    tc::grid_dep_wait();  // launched with programmatic stream serialisation
    tc::grid_dep_launch();
    constexpr int VE = 16 / (int)sizeof(T), LPT = kD / VE;  // elements per load, lanes per token
    static_assert(32 % LPT == 0, "a token's lanes share a warp");
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long tok = g / LPT;
    const int sub = (int)(g % LPT);
    const bool in = tok < (long long)BH * ld;
    const int bh = in ? (int)(tok / ld) : 0, t = in ? (int)(tok % ld) : 0;
    float s = 0.f;
    if (in && t < L && (mask == nullptr || mask[(size_t)(bh / H) * L + t])) {
        const size_t o = ((size_t)bh * L + t) * kD + (size_t)sub * VE;
        float x[8], y[8];
        load_vec(X + o, x, VE);
        load_vec(Y + o, y, VE);
#pragma unroll
        for (int e = 0; e < VE; ++e) s = fmaf(x[e], y[e], s);
    }
#pragma unroll
    for (int off = LPT / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off, LPT);
    if (in && sub == 0) out[(size_t)bh * ld + t] = s;
}

// eu[a][bh][t] = exp(u^(a) - u^(R)), ev[a][bh][t] = exp(v^(a) - v^(R)), a = 0..R;
// zero on masked tokens.  state: [BH][2R+2][ld].
__global__ void k_orbit(const float* state, int R, int L, int H, int ld, int BH,
                        const uint8_t* mask, float* eu, float* ev, size_t vstride) {
    tc::grid_dep_wait();  // launched with programmatic stream serialisation
    tc::grid_dep_launch();
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= (long long)BH * ld) return;
    const int bh = (int)(g / ld), t = (int)(g % ld);
    const bool ok = t >= L || mask == nullptr || mask[(size_t)(bh / H) * L + t];
    const float* st = state + (size_t)bh * (2 * R + 2) * ld;
    const float uR = st[(size_t)(2 * R) * ld + t], vR = st[(size_t)(2 * R + 1) * ld + t];
    for (int a = 0; a <= R; ++a) {
        const float ua = st[(size_t)(2 * a) * ld + t], va = st[(size_t)(2 * a + 1) * ld + t];
        eu[a * vstride + g] = ok ? ex2((ua - uR) * kLog2e) : 0.f;
        ev[a * vstride + g] = ok ? ex2((va - vR) * kLog2e) : 0.f;
    }
}

// out = s * x * y elementwise over BH*ld (x or y null means 1).
__global__ void k_vmul(const float* x, const float* y, float s, float* out, long long n) {
    tc::grid_dep_wait();  // launched with programmatic stream serialisation
    tc::grid_dep_launch();
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n) return;
    float v = s;
    if (x) v *= x[g];
    if (y) v *= y[g];
    out[g] = v;
}

// Working copy of state rows [r_lo, r_hi) of every problem: w = log2(e) * dual
// on valid tokens, -inf on masked ones (state [BH][2R+2][ld], work [BH][2R+2][L]),
// and the operand rows aug [BH][2R+2][L][16] (see tcr::put_aug).
__global__ void k_work(const float* state, int nrows, int ld, int L, int H, int BH,
                       const uint8_t* mask, int r_lo, int r_hi, float inv_c, float* work,
                       __nv_bfloat16* aug, int* status) {
    tc::grid_dep_wait();  // launched with programmatic stream serialisation
    tc::grid_dep_launch();
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int nr = r_hi - r_lo;
    if (g >= (long long)BH * nr * L) return;
    const int t = (int)(g % L);
    const long long rest = g / L;
    const int row = r_lo + (int)(rest % nr), bh = (int)(rest / nr);
    if (!SA_BOUNDS(bh < BH && row < nrows, status)) return;
    const bool ok = mask == nullptr || mask[(size_t)(bh / H) * L + t];
    const float v = state[((size_t)bh * nrows + row) * ld + t];
    const size_t o = ((size_t)bh * nrows + row) * L + t;
    work[o] = ok ? v * kLog2e : -INFINITY;
    tcr::put_aug(aug + o * 16, ok, v * inv_c);
}

// dv_dust[h][e] = sum_b part[(b*H + h)][e]
__global__ void k_dvd_reduce(const float* part, int B, int H, float* out) {
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= H * kD) return;
    const int h = g / kD, e = g % kD;
    float s = 0.f;
    for (int b = 0; b < B; ++b) s += part[((size_t)b * H + h) * kD + e];
    out[g] = s;
}

// Cotangent of the dustbin score (one learned dustbin token): the score enters
// every dustbin entry -- column (i, L), row (L, j) and the corner (L, L) -- so
// its cotangent is the sum of dS over them, each entry's staircase plans formed
// by their own exponential:
//   dS_e = P^(R,R)_e (G_e - vbar^R_col) - sum_{r=1..R} P^(r,r-1)_e ubar^r_row
//          - sum_{r=1..R-1} P^(r,r)_e vbar^r_col,   P^(a,b)_e = exp(s + u^(a)_row + v^(b)_col)
// with G_(i,L) = <dO_i, v_dust> and G = 0 on the dustbin row (it has no
// output).  R = 0 keeps every dual constant: dS_e = P_e G_e.  The entries
// cancel to a remainder far smaller than their sizes, so the sums run in
// double.  One block per problem writes its sum to part[bh]; ubar/vbar hold
// index r at r * rs floats.
template <typename T>
__global__ void k_dscore(const T* dO, const float* v_dust, const uint8_t* mask,
                         const float* state, const float* ubar, const float* vbar, size_t rs,
                         int R, int L, int H, int ld, float sd, double* part) {
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const float* st = state + (size_t)bh * (2 * R + 2) * ld;
    auto U = [&](int a, int t) { return st[(size_t)(2 * a) * ld + t]; };
    auto V = [&](int a, int t) { return st[(size_t)(2 * a + 1) * ld + t]; };
    auto UB = [&](int r, int t) { return ubar[(size_t)r * rs + (size_t)bh * ld + t]; };
    auto VB = [&](int r, int t) { return vbar[(size_t)r * rs + (size_t)bh * ld + t]; };
    // dS at (row i, column j) without the A term
    auto ds_tail = [&](int i, int j) {
        if (R == 0) return 0.0;
        double g = -(double)expf(sd + U(R, i) + V(R, j)) * VB(R, j);
        for (int r = 1; r <= R; ++r) g -= (double)expf(sd + U(r, i) + V(r - 1, j)) * UB(r, i);
        for (int r = 1; r < R; ++r) g -= (double)expf(sd + U(r, i) + V(r, j)) * VB(r, j);
        return g;
    };
    double acc = 0.0;
    for (int t = threadIdx.x; t < L; t += blockDim.x) {
        if (mask && !mask[(size_t)b * L + t]) continue;
        float gi = 0.f;  // <dO_t, v_dust>
        if (v_dust) {
            const T* row = dO + ((size_t)bh * L + t) * kD;
            const float* vd = v_dust + (size_t)h * kD;
            for (int e = 0; e < kD; ++e) gi = fmaf(to_f32(row[e]), vd[e], gi);
        }
        acc += (double)expf(sd + U(R, t) + V(R, L)) * gi + ds_tail(t, L) + ds_tail(L, t);
    }
    if (threadIdx.x == 0) acc += ds_tail(L, L);
    __shared__ double red[32];
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double sum = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) sum += red[w];
        part[bh] = sum;
    }
}

// out[i] += in[i], i < n.
__global__ void k_add(float* out, const float* in, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] += in[i];
}

// out[0] = sum of part[0..n) in a fixed order (one block of 256 threads).
__global__ void k_sum_parts(const double* part, int n, float* out) {
    __shared__ double red[256];
    double s = 0.0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) s += part[i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) out[0] = (float)red[0];
}

// The dS sweep's modifier as K16 operands of the dO V^T contraction, for both
// sweeps at once: out[i][bh][t][16] bf16, i = row side of q, column side of k,
// row side of k, column side of q.  Slots 3k, 3k+1, 3k+2 of term k < n hold the
// bf16 halves (hi, hi, lo) of the term's vector for a row side and (hi, lo, hi)
// for a column side (a null vector: 1); the other slots are 0.
struct AugTerms {
    Vec q[4], k[4];  // the terms' query-side and key-side vectors
    int n;
    __nv_bfloat16* out[4];
};
__device__ __forceinline__ void put_aug_row(const Vec (&v)[4], int n, bool row, int bh, int t,
                                            __nv_bfloat16* dst) {
    uint16_t sl[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) sl[i] = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if (k >= n) break;
        const float x = v[k].p ? v[k].at(bh, t) : 1.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
        const uint16_t h = __bfloat16_as_ushort(hi), l = __bfloat16_as_ushort(lo);
        sl[3 * k] = h;
        sl[3 * k + 1] = row ? h : l;
        sl[3 * k + 2] = row ? l : h;
    }
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = (uint32_t)sl[2 * i] | ((uint32_t)sl[2 * i + 1] << 16);
    uint4* o = reinterpret_cast<uint4*>(dst);
    o[0] = make_uint4(w[0], w[1], w[2], w[3]);
    o[1] = make_uint4(w[4], w[5], w[6], w[7]);
}
__global__ void k_aug(AugTerms tm, int L, int BH) {
    tc::grid_dep_wait();  // launched with programmatic stream serialisation
    tc::grid_dep_launch();
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= (long long)BH * L) return;
    const int bh = (int)(g / L), t = (int)(g % L);
    put_aug_row(tm.q, tm.n, true, bh, t, tm.out[0] + (size_t)g * 16);
    put_aug_row(tm.k, tm.n, false, bh, t, tm.out[1] + (size_t)g * 16);
    put_aug_row(tm.k, tm.n, true, bh, t, tm.out[2] + (size_t)g * 16);
    put_aug_row(tm.q, tm.n, false, bh, t, tm.out[3] + (size_t)g * 16);
}

// out[0] += sum_i (x_i - y_i)^2, out[1] += sum_i y_i^2 in double: grid-stride
// loop, warp shuffles, one atomic pair per warp.
template <typename T>
__global__ void k_sq_dist(const T* x, const T* y, long long n, double* out) {
    double s0 = 0.0, s1 = 0.0;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const double a = to_f32(x[i]), b = to_f32(y[i]);
        s0 += (a - b) * (a - b);
        s1 += b * b;
    }
    for (int o = 16; o > 0; o >>= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    }
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(out, s0);
        atomicAdd(out + 1, s1);
    }
}

// A wait that nothing completes: thread 0 waits on a fresh mbarrier (one
// expected arrival, none made) for `budget` cycles through the library's
// bounded wait, then records the timeout like any stalled pipeline stage.
__global__ void k_stall(int* status, long long budget) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0, budget))
        atomicCAS(status, (int)SA_OK, (int)SA_ERR_TIMEOUT);
    __syncthreads();
}

// The two exponentials of the row-sum sweeps side by side (test hook): y_poly
// from the FMA-pipe polynomial, y_mufu from ex2.approx, of each x <= 0.
__global__ void k_exp2_pair(const float* x, long long n, float* y_poly, float* y_mufu) {
    const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
    float e0, e1;
    tcr::exp2_poly2(x0, x1, e0, e1);
    y_poly[i] = e0;
    y_mufu[i] = ex2(x0);
    if (i + 1 < n) {
        y_poly[i + 1] = e1;
        y_mufu[i + 1] = ex2(x1);
    }
}

// Sets the status word when any element is NaN or Inf.
template <typename T>
__global__ void k_finite(const T* x, long long n, int* status) {
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    bool bad = false;
    for (long long i = g; i < n; i += (long long)gridDim.x * blockDim.x)
        if (!isfinite(to_f32(x[i]))) bad = true;
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
        atomicCAS(status, (int)SA_OK, (int)SA_ERR_NONFINITE);
}

// P^(a,b) in band layout; scores with the same fp32 FMA order as the sweeps.
template <typename T>
__global__ void k_debug_plan(const T* q, const T* k, const uint8_t* mask, const float* state,
                             int a, int b, int R, int L, int H, int W, int ld, float c2,
                             int dustbin, float sd2, float* band, float* dcol, float* drow) {
    const int bh = blockIdx.y;
    const int i = blockIdx.x;
    const int bw = 2 * W + 1;
    const uint8_t* mk = mask ? mask + (size_t)(bh / H) * L : nullptr;
    const float* st = state + (size_t)bh * (2 * R + 2) * ld;
    const float* ua = st + (size_t)(2 * a) * ld;
    const float* vb = st + (size_t)(2 * b + 1) * ld;
    if (i == L) {  // dustbin row
        if (!dustbin || !drow) return;
        for (int j = threadIdx.x; j <= L; j += blockDim.x) {
            float v = 0.f;
            if (j == L || !mk || mk[j]) v = ex2(sd2 + (ua[L] + vb[j]) * kLog2e);
            drow[(size_t)bh * (L + 1) + j] = v;
        }
        return;
    }
    const bool vi = !mk || mk[i];
    const T* qi = q + ((size_t)bh * L + i) * kD;
    for (int t = threadIdx.x; t < bw; t += blockDim.x) {
        const int j = i - W + t;
        float v = 0.f;
        if (vi && j >= 0 && j < L && (!mk || mk[j])) {
            const T* kj = k + ((size_t)bh * L + j) * kD;
            float acc = 0.f;
            for (int e = 0; e < kD; ++e) acc = fmaf(to_f32(qi[e]), to_f32(kj[e]), acc);
            v = ex2(fmaf(c2, acc, (ua[i] + vb[j]) * kLog2e));
        }
        band[((size_t)bh * L + i) * bw + t] = v;
    }
    if (dustbin && dcol && threadIdx.x == 0)
        dcol[(size_t)bh * L + i] = vi ? ex2(sd2 + (ua[i] + vb[L]) * kLog2e) : 0.f;
}

// ---------------------------------------------------------------------------
// launch helpers
// ---------------------------------------------------------------------------

// Optional launch trace (sa_params.trace_*): caller-owned CUDA events recorded
// on the call's stream around each kernel launch.
struct Tracer {
    const sa_params* p = nullptr;
    cudaStream_t st = nullptr;
    int n = 0;
    bool on() const { return p->trace_events && p->trace_cap > 0 && n < p->trace_cap; }
    void begin(int kind) {
        if (!on()) return;
        cudaEventRecord((cudaEvent_t)p->trace_events[2 * n], st);
        if (p->trace_kinds) p->trace_kinds[n] = kind;
    }
    void end() {
        if (on()) cudaEventRecord((cudaEvent_t)p->trace_events[2 * n + 1], st);
        ++n;
        if (p->trace_count) *p->trace_count = n;
    }
};

constexpr int kind_of(int mode) {
    return mode == simt::LSE ? SA_KERNEL_LSE_SWEEP
         : mode == simt::PV ? SA_KERNEL_PV
         : mode == simt::WSUM ? SA_KERNEL_WSUM : SA_KERNEL_DS;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// [BH][L][64] bf16 viewed as a 3-D tensor; 64 x 128 x 1 boxes, 128-byte swizzle,
// zero fill outside the tensor (rows < 0 or >= L).
bool make_map(CUtensorMap* m, const void* ptr, int L, int BH) {
    auto fn = encode_tiled();
    if (!fn || !ptr) return false;
    cuuint64_t dims[3] = {64, (cuuint64_t)L, (cuuint64_t)BH};
    cuuint64_t strides[2] = {64 * 2, (cuuint64_t)L * 64 * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// [BH][L][16] bf16 (the dS modifier's K16 operands), 128-token boxes, 32-byte swizzle
bool make_map_aug(CUtensorMap* m, const void* ptr, int L, int BH) {
    auto fn = encode_tiled();
    if (!fn || !ptr) return false;
    cuuint64_t dims[3] = {16, (cuuint64_t)L, (cuuint64_t)BH};
    cuuint64_t strides[2] = {16 * 2, (cuuint64_t)L * 16 * 2};
    cuuint32_t box[3] = {16, 128, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// [BH][L][16] bf16 operand rows whose problems lie `bh_stride` elements apart
bool make_map_aug_strided(CUtensorMap* m, const void* ptr, int L, int BH, long long bh_stride) {
    auto fn = encode_tiled();
    if (!fn || !ptr) return false;
    cuuint64_t dims[3] = {16, (cuuint64_t)L, (cuuint64_t)BH};
    cuuint64_t strides[2] = {16 * 2, (cuuint64_t)bh_stride * 2};
    cuuint32_t box[3] = {16, 128, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// SMs of the device (persistent grids take one or two CTAs per SM); read once
// from the first device asked, since the library targets a single GPU model
// (sm_100a)
int sm_count() {
    static int nsm = 0;
    if (nsm == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
            nsm = 148;
    }
    return nsm;
}

// Launches a persistent sweep with programmatic stream serialisation: its
// CTAs may be placed while the previous kernel of the stream finishes, so their
// set-up (barrier init, TMEM allocation) overlaps its tail; the sweeps wait for
// that kernel (griddepcontrol.wait) before any global access, so the ordering
// of their reads and writes is that of a plain launch.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <int MODE, bool ONLINE, int NT>
cudaError_t launch_tc(const simt::SweepArgs& a, int BH, cudaStream_t st, Tracer& tr,
                      int* status) {
    tcs::Maps maps;
    std::memset(&maps, 0, sizeof(maps));
    bool ok = make_map(&maps.A, a.A, a.L, BH) && make_map(&maps.B, a.Bo, a.L, BH);
    if (tcs::is_ds(MODE)) ok = ok && make_map(&maps.A2, a.A2, a.L, BH) && make_map(&maps.B2, a.B2, a.L, BH);
    if (MODE == simt::PV) ok = ok && make_map(&maps.X, a.X, a.L, BH);
    if (tcs::aug(MODE, NT))
        ok = ok && make_map_aug(&maps.AR, a.aug_row, a.L, BH) && make_map_aug(&maps.AC, a.aug_col, a.L, BH);
    if (tcs::augs(MODE)) {  // the constant row-block operand and the column duals' rows
        void* ones = nullptr;
        ok = ok && cudaGetSymbolAddress(&ones, tcr::g_aug_ones) == cudaSuccess && ones &&
             make_map_aug_strided(&maps.AR, ones, 128, 1, 128 * 16) &&
             make_map_aug_strided(&maps.AC, a.augc, a.L, BH, a.aug_s);
    }
    if (!ok) return cudaErrorInvalidValue;
    // persistent: one CTA per SM (two for the online LSE sweep), each a contiguous tile range
    const long long ntiles = (long long)((a.L + 127) / 128) * BH;
    const dim3 grid((unsigned)std::min<long long>(ntiles, (long long)sm_count() * tcs::ctas_per_sm(MODE)));
    const int smem = tcs::smem_bytes(MODE, NT);
    cudaError_t e = cudaFuncSetAttribute(tcs::tc_band_sweep<MODE, ONLINE, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    tr.begin(kind_of(MODE));
    e = launch_pdl(tcs::tc_band_sweep<MODE, ONLINE, NT>, grid, dim3(tcs::nthreads(MODE)), smem, st, a, maps,
                   status, BH);
    tr.end();
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Exponentials of every 32 entries of a row-sum sweep's in-band group that run
// on the FMA pipe (the rest on the MUFU unit).
// Exponentials per 32 on the FMA pipe (the rest on MUFU) in the row-sum sweeps'
// in-band groups: measured on long32k, 8 of 32 takes 1-4 % off an LSE sweep
// (W 256-320) and slows WSUM, whose epilogue has more FMA work of its own.
#ifndef SA_ROWSUM_KP_LSE
#define SA_ROWSUM_KP_LSE 8
#endif
#ifndef SA_ROWSUM_KP_WSUM
#define SA_ROWSUM_KP_WSUM 0
#endif

// The row-sum sweeps (shifted LSE, WSUM) on the tensor cores: persistent, one
// CTA per SM.
template <int MODE>
cudaError_t launch_rowsum(const simt::SweepArgs& a, int BH, cudaStream_t st, Tracer& tr,
                          int* status) {
    tcr::Maps maps;
    std::memset(&maps, 0, sizeof(maps));
    void* ones = nullptr;
    if (cudaGetSymbolAddress(&ones, tcr::g_aug_ones) != cudaSuccess || !ones) return cudaErrorInvalidValue;
    if (!make_map(&maps.A, a.A, a.L, BH) || !make_map(&maps.B, a.Bo, a.L, BH) ||
        !make_map_aug_strided(&maps.BA, a.augc, a.L, BH, a.aug_s) ||
        !make_map_aug_strided(&maps.AO, ones, 128, 1, 128 * 16))
        return cudaErrorInvalidValue;
    const long long ntiles = (long long)((a.L + 127) / 128) * BH;
    const dim3 grid((unsigned)std::min<long long>(ntiles, (long long)sm_count()));
    auto kern = tcr::tc_rowsum_sweep<MODE, MODE == simt::LSE ? SA_ROWSUM_KP_LSE : SA_ROWSUM_KP_WSUM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         tcr::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    tr.begin(kind_of(MODE));
    e = launch_pdl(kern, grid, dim3(tcr::NTHREADS), tcr::SMEM_BYTES, st, a, maps, status, BH);
    tr.end();
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename T, int MODE>
cudaError_t launch_sweep(const simt::SweepArgs& a, int BH, cudaStream_t st, Tracer& tr,
                         int* status) {
    // bf16 storage without a dustbin runs on the tensor cores
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        if (!a.dustbin) {
            if constexpr (MODE == simt::LSE) {
                if (a.online) return launch_tc<MODE, true, 0>(a, BH, st, tr, status);
                return launch_rowsum<MODE>(a, BH, st, tr, status);
            } else if constexpr (MODE == simt::WSUM) {
                return launch_rowsum<MODE>(a, BH, st, tr, status);
            } else if constexpr (MODE == simt::DS1 || MODE == simt::DSD) {
                if (MODE == simt::DS1 && a.nterms == 0)  // R = 0: dS = P * G
                    return launch_tc<MODE, false, 0>(a, BH, st, tr, status);
                switch (a.nterms) {  // a block of the 2R terms: 2, 4, 6 or MAXT
                    case 2: return launch_tc<MODE, false, 2>(a, BH, st, tr, status);
                    case 4: return launch_tc<MODE, false, 4>(a, BH, st, tr, status);
                    case 6: return launch_tc<MODE, false, 6>(a, BH, st, tr, status);
                    case 8: return launch_tc<MODE, false, 8>(a, BH, st, tr, status);
                    default: return cudaErrorInvalidValue;
                }
            } else {
                return launch_tc<MODE, false, 0>(a, BH, st, tr, status);
            }
        }
    }
    const int nblk = (a.L + simt::BM - 1) / simt::BM;
    const dim3 grid(nblk + (a.dust_cta ? 1 : 0), BH);
    const size_t smem = (size_t)simt::smem_floats(MODE) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(simt::band_sweep<T, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    tr.begin(kind_of(MODE));
    simt::band_sweep<T, MODE><<<grid, simt::NT, smem, st>>>(a);
    tr.end();
    return cudaGetLastError();
}

#define SA_AUX(tr, ...)                        \
    do {                                       \
        (tr).begin(SA_KERNEL_AUX);             \
        __VA_ARGS__;                           \
        (tr).end();                            \
        SA_CUDA(cudaGetLastError());           \
    } while (0)

Vec vec(const float* p, long long s) { return Vec{p, s}; }
MVec mvec(float* p, long long s) { return MVec{p, s}; }

struct Ctx {
    const sa_params* p;
    Dims d;
    cudaStream_t st;
    float c;     // natural score scale 1/(sqrt(d) eps)
    long long sst;  // per-bh stride of a state row: (2R+2)*ld
    const float* state;
    int* status;   // device status word (workspace header)
    mutable Tracer tr;
    const sa_shard* shard = nullptr;  // sequence-sharded call, else null
    // state row r (0..2R+1) as a Vec
    Vec srow(int r) const { return vec(state + (size_t)r * d.ld, sst); }
    // its working copy and operand row (tensor-core row-sum sweeps), or null
    float* work = nullptr;
    __nv_bfloat16* waug = nullptr;
    Vec wrow(int r) const {
        return work ? vec(work + (size_t)r * d.L, (long long)(2 * d.R + 2) * d.L) : Vec{nullptr, 0};
    }
    MVec mwrow(int r) const { Vec v = wrow(r); return MVec{const_cast<float*>(v.p), v.s}; }
    __nv_bfloat16* augrow(int r) const { return waug ? waug + (size_t)r * d.L * 16 : nullptr; }
    long long aug_stride() const { return (long long)(2 * d.R + 2) * d.L * 16; }
    void set_work(char* base) {
        work = (float*)base;
        waug = (__nv_bfloat16*)(base + work_floats_bytes(d));
    }
    // rebuilds working rows [lo, hi) from the state
    sa_status refresh_work(const uint8_t* mask, int lo, int hi) const {
        if (!work) return SA_OK;
        const long long n = (long long)d.BH * (hi - lo) * d.L;
        tr.begin(SA_KERNEL_AUX);
        const cudaError_t e = launch_pdl(k_work, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, state,
                                         2 * d.R + 2, d.ld, d.L, d.H, d.BH, mask, lo, hi, 1.0f / c, work,
                                         waug, status);
        tr.end();
        return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? SA_OK : SA_ERR_CUDA;
    }
    // sharded calls: the neighbours' values into the halo entries of a vector
    // just produced (rows of d.L entries, row_stride apart)
    sa_status halo(const float* v, long long row_stride) const {
        if (!shard) return SA_OK;
        return shard->exchange(const_cast<float*>(v), row_stride, d.BH, shard->user, st) == 0
                   ? SA_OK
                   : SA_ERR_EXCHANGE;
    }
};

#define SA_HALO(x, v, stride)                      \
    do {                                           \
        sa_status h_ = (x).halo((v), (stride));    \
        if (h_ != SA_OK) return h_;                \
    } while (0)

simt::SweepArgs base_args(const Ctx& x) {
    simt::SweepArgs a;
    std::memset(&a, 0, sizeof(a));
    a.L = x.d.L;
    a.W = x.p->W;
    a.H = x.d.H;
    a.ld = x.d.ld;
    a.c2 = x.c * kLog2e;
    a.dustbin = x.p->dustbin;
    a.dust_cta = x.p->dustbin;
    a.sd2 = x.p->dustbin ? x.p->dustbin_score * kLog2e : 0.f;
    a.sgn = 1.f;
    a.out_scale = x.c;
    a.status = x.status;
    return a;
}

#define SA_CUDA(call)                              \
    do {                                           \
        cudaError_t e_ = (call);                   \
        if (e_ != cudaSuccess) return SA_ERR_CUDA; \
    } while (0)

template <typename T>
sa_status fwd_impl(const Ctx& x, const T* q, const T* k, const T* v, const uint8_t* mask,
                   const float* v_dust, T* o, float* state) {
    const Dims& d = x.d;
    // v0 = 0 and u0 = 0 (u0 stays 0 when T == 0)
    SA_CUDA(cudaMemsetAsync(state, 0, (size_t)d.BH * (2 * d.R + 2) * d.ld * sizeof(float), x.st));
    sa_status s = x.refresh_work(mask, 1, 2);  // v0's working copy
    if (s != SA_OK) return s;
    simt::SweepArgs a = base_args(x);
    a.mask = mask;
    const int iters = x.p->T + d.R;
    for (int it = 0; it < iters; ++it) {
        const int rin = it < x.p->T ? 0 : it - x.p->T;       // v index read
        const int rout = it < x.p->T ? 0 : it - x.p->T + 1;  // u, v index written
        // rows: u^(rout) = -LSE_j(S + v^(rin)); the previous u (u^(rin), or u0 in
        // place during the base) is the exponent shift, except on the first update
        a.A = q; a.Bo = k;
        a.cd = x.srow(2 * rin + 1);
        a.rd = x.srow(2 * rin);
        a.cdw = x.wrow(2 * rin + 1);
        a.rdw = x.wrow(2 * rin);
        a.outw = x.mwrow(2 * rout);
        a.augc = x.augrow(2 * rin + 1);
        a.augo = x.augrow(2 * rout);
        a.aug_s = x.aug_stride();
        a.online = (it == 0);
        a.out_vec = mvec(state + (size_t)(2 * rout) * d.ld, x.sst);
        SA_CUDA((launch_sweep<T, simt::LSE>(a, d.BH, x.st, x.tr, x.status)));
        SA_HALO(x, a.out_vec.p, x.sst);
        // the first update (a running max, no working copy) and sharded calls
        // (the exchange refills the state's halo entries) renew the working copy
        if (it == 0 || x.shard) {
            s = x.refresh_work(mask, 2 * rout, 2 * rout + 1);
            if (s != SA_OK) return s;
        }
        // columns: v^(rout) = -LSE_i(S + u^(rout)), shifted by the previous v
        a.A = k; a.Bo = q;
        a.cd = x.srow(2 * rout);
        a.rd = x.srow(2 * rin + 1);
        a.cdw = x.wrow(2 * rout);
        a.rdw = x.wrow(2 * rin + 1);
        a.outw = x.mwrow(2 * rout + 1);
        a.augc = x.augrow(2 * rout);
        a.augo = x.augrow(2 * rout + 1);
        a.aug_s = x.aug_stride();
        a.online = 0;
        a.out_vec = mvec(state + (size_t)(2 * rout + 1) * d.ld, x.sst);
        SA_CUDA((launch_sweep<T, simt::LSE>(a, d.BH, x.st, x.tr, x.status)));
        SA_HALO(x, a.out_vec.p, x.sst);
        if (x.shard) {
            s = x.refresh_work(mask, 2 * rout + 1, 2 * rout + 2);
            if (s != SA_OK) return s;
        }
    }
    // O = P^(R,R) V (+ dustbin column times v_dust)
    simt::SweepArgs b = base_args(x);
    b.mask = mask;
    b.dust_cta = 0;
    b.A = q; b.Bo = k; b.X = v;
    b.Xd = v_dust;
    b.rd = x.srow(2 * d.R);
    b.cd = x.srow(2 * d.R + 1);
    b.cdw = x.wrow(2 * d.R + 1);
    b.augc = x.augrow(2 * d.R + 1);
    b.aug_s = x.aug_stride();
    b.out_mat = o;
    SA_CUDA((launch_sweep<T, simt::PV>(b, d.BH, x.st, x.tr, x.status)));
    return SA_OK;
}

template <typename T>
sa_status bwd_impl(const Ctx& x, const T* q, const T* k, const T* v, const uint8_t* mask,
                   const float* v_dust, const T* o, const T* dO, T* dq, T* dk, T* dv,
                   float* dv_dust, float* d_score, char* ws) {
    const Dims& d = x.d;
    const int R = d.R;
    const BwdLayout l = bwd_layout(d, x.p);
    const long long vs = d.ld;  // per-bh stride of a workspace vector
    const size_t vstride = l.vec / sizeof(float);
    auto W_ = [&](size_t off, int idx) { return (float*)(ws + off + (size_t)idx * l.vec); };
    float* A_ = W_(l.a, 0);
    float* dvd = (float*)(ws + l.dvd);
    const long long nvec = (long long)d.BH * d.ld;
    const int eb = 256;
    const unsigned egrid = (unsigned)((nvec + eb - 1) / eb);
    const bool direct = x.p->bwd == SA_BWD_DIRECT;

    // the working copy of the whole state (read by the row-sum sweeps)
    {
        const sa_status s = x.refresh_work(mask, 0, 2 * R + 2);
        if (s != SA_OK) return s;
    }
    // a = rowdot(dO, O); orbit factors
    {
        const long long thr = nvec * (kD / (16 / (long long)sizeof(T)));
        SA_AUX(x.tr, SA_CUDA(launch_pdl(k_rowdot<T>, dim3((unsigned)((thr + 255) / 256)), dim3(256), 0,
                                        x.st, dO, o, mask, d.L, d.H, d.ld, d.BH, A_)));
        SA_AUX(x.tr, SA_CUDA(launch_pdl(k_orbit, dim3(egrid), dim3(eb), 0, x.st, x.state, R, d.L, d.H,
                                        d.ld, d.BH, mask, W_(l.eu, 0), W_(l.ev, 0), vstride)));
    }
    const Vec uR = x.srow(2 * R), vR = x.srow(2 * R + 1);
    auto U = [&](int r) { return x.srow(2 * r); };
    auto V = [&](int r) { return x.srow(2 * r + 1); };
    auto ub = [&](int r) { return W_(l.ubar, r); };
    auto vb = [&](int r) { return W_(l.vbar, r); };
    auto eu = [&](int r) { return W_(l.eu, r); };
    auto ev = [&](int r) { return W_(l.ev, r); };

    // dV = P^T dO, vbar^R = rowdot(V, dV)  (key sweep; dustbin row: dv_dust partials)
    {
        simt::SweepArgs a = base_args(x);
        a.mask = mask;
        a.A = k; a.Bo = q; a.X = dO; a.Y = v;
        a.Yd = v_dust;
        a.rd = vR; a.cd = uR;
        a.cdw = x.wrow(2 * R);
        a.augc = x.augrow(2 * R);
        a.aug_s = x.aug_stride();
        a.out_mat = dv;
        a.out_vec = mvec(vb(R), vs);
        a.dvd_part = dvd;
        SA_CUDA((launch_sweep<T, simt::PV>(a, d.BH, x.st, x.tr, x.status)));
        if (R > 0) SA_HALO(x, vb(R), vs);
    }
    // ubar^R = a - P vbar^R  (query sweep; R = 0 has no dual cotangents)
    if (R > 0) {
        simt::SweepArgs a = base_args(x);
        a.mask = mask;
        a.A = q; a.Bo = k;
        a.rd = uR; a.cd = vR;
        a.rdw = x.wrow(2 * R); a.cdw = x.wrow(2 * R + 1);
        a.augc = x.augrow(2 * R + 1); a.aug_s = x.aug_stride();
        a.w = vec(vb(R), vs);
        a.base = vec(A_, vs);
        a.sgn = -1.f;
        a.out_vec = mvec(ub(R), vs);
        SA_CUDA((launch_sweep<T, simt::WSUM>(a, d.BH, x.st, x.tr, x.status)));
        SA_HALO(x, ub(R), vs);
    }
    for (int r = R; r >= 2; --r) {
        // vbar^(r-1) = -P^(r,r-1)^T ubar^r
        simt::SweepArgs a = base_args(x);
        a.mask = mask;
        a.A = k; a.Bo = q;
        a.sgn = -1.f;
        a.out_vec = mvec(vb(r - 1), vs);
        if (direct) {
            a.rd = V(r - 1); a.cd = U(r);
            a.rdw = x.wrow(2 * (r - 1) + 1); a.cdw = x.wrow(2 * r);
            a.augc = x.augrow(2 * r); a.aug_s = x.aug_stride();
            a.w = vec(ub(r), vs);
        } else {
            SA_AUX(x.tr, SA_CUDA(launch_pdl(k_vmul, dim3(egrid), dim3(eb), 0, x.st,
                                 eu(r), ub(r), 1.f, W_(l.w, 0), nvec)));
            a.rd = vR; a.cd = uR;
            a.rdw = x.wrow(2 * R + 1); a.cdw = x.wrow(2 * R);
            a.augc = x.augrow(2 * R); a.aug_s = x.aug_stride();
            a.w = vec(W_(l.w, 0), vs);
            a.mult = vec(ev(r - 1), vs);
        }
        SA_CUDA((launch_sweep<T, simt::WSUM>(a, d.BH, x.st, x.tr, x.status)));
        SA_HALO(x, vb(r - 1), vs);
        // ubar^(r-1) = -P^(r-1,r-1) vbar^(r-1)
        simt::SweepArgs b = base_args(x);
        b.mask = mask;
        b.A = q; b.Bo = k;
        b.sgn = -1.f;
        b.out_vec = mvec(ub(r - 1), vs);
        if (direct) {
            b.rd = U(r - 1); b.cd = V(r - 1);
            b.rdw = x.wrow(2 * (r - 1)); b.cdw = x.wrow(2 * (r - 1) + 1);
            b.augc = x.augrow(2 * (r - 1) + 1); b.aug_s = x.aug_stride();
            b.w = vec(vb(r - 1), vs);
        } else {
            SA_AUX(x.tr, SA_CUDA(launch_pdl(k_vmul, dim3(egrid), dim3(eb), 0, x.st,
                                 ev(r - 1), vb(r - 1), 1.f, W_(l.w, 0), nvec)));
            b.rd = uR; b.cd = vR;
            b.rdw = x.wrow(2 * R); b.cdw = x.wrow(2 * R + 1);
            b.augc = x.augrow(2 * R + 1); b.aug_s = x.aug_stride();
            b.w = vec(W_(l.w, 0), vs);
            b.mult = vec(eu(r - 1), vs);
        }
        SA_CUDA((launch_sweep<T, simt::WSUM>(b, d.BH, x.st, x.tr, x.status)));
        SA_HALO(x, ub(r - 1), vs);
    }

    // modifier / staircase terms, query side (rq) and key side (rk)
    //   one reference:  M = G + sum_k rq_k[i] rk_k[j]
    //     k=0: (1, -vbar^R);  r=1..R: (-eu^r ubar^r, ev^(r-1));  r=1..R-1: (-eu^r, ev^r vbar^r)
    //   direct: dS = sum_k exp(S + eq_k[i] + ek_k[j]) (g_k G + cq_k[i] + ck_k[j])
    //     k=0: (u^R, v^R; G - vbar^R);  r: (u^r, v^(r-1); -ubar^r);  r<R: (u^r, v^r; -vbar^r)
    int nt = 0;
    std::vector<Vec> rq(2 * R), rk(2 * R), eq(2 * R), ek(2 * R), cq(2 * R), ck(2 * R);
    std::vector<float> gk(2 * R);
    const Vec none{nullptr, 0};
    auto slot_q = [&](int i) { return (float*)(ws + l.rv + (size_t)i * l.vec); };
    auto slot_k = [&](int i) { return (float*)(ws + l.cv + (size_t)i * l.vec); };
    if (R > 0) {  // R = 0: every dual is a constant and dS = P * G (no terms)
        // k = 0
        SA_AUX(x.tr, SA_CUDA(launch_pdl(k_vmul, dim3(egrid), dim3(eb), 0, x.st,
                             vb(R), nullptr, -1.f, slot_k(0), nvec)));
        rq[nt] = none; rk[nt] = vec(slot_k(0), vs);
        eq[nt] = uR; ek[nt] = vR; cq[nt] = none; ck[nt] = vec(slot_k(0), vs); gk[nt] = 1.f;
        ++nt;
        for (int r = 1; r <= R; ++r) {
            if (direct) {
                SA_AUX(x.tr, SA_CUDA(launch_pdl(k_vmul, dim3(egrid), dim3(eb), 0, x.st,
                                     ub(r), nullptr, -1.f, slot_q(nt), nvec)));
            } else {
                SA_AUX(x.tr, SA_CUDA(launch_pdl(k_vmul, dim3(egrid), dim3(eb), 0, x.st,
                                     eu(r), ub(r), -1.f, slot_q(nt), nvec)));
            }
            rq[nt] = vec(slot_q(nt), vs); rk[nt] = vec(ev(r - 1), vs);
            eq[nt] = U(r); ek[nt] = V(r - 1); cq[nt] = vec(slot_q(nt), vs); ck[nt] = none;
            gk[nt] = 0.f;
            ++nt;
        }
        for (int r = 1; r < R; ++r) {
            if (direct) {
                SA_AUX(x.tr, SA_CUDA(launch_pdl(k_vmul, dim3(egrid), dim3(eb), 0, x.st,
                                     vb(r), nullptr, -1.f, slot_k(nt), nvec)));
                eq[nt] = U(r); ek[nt] = V(r); cq[nt] = none; ck[nt] = vec(slot_k(nt), vs);
                gk[nt] = 0.f;
            } else {
                SA_AUX(x.tr, SA_CUDA(launch_pdl(k_vmul, dim3(egrid), dim3(eb), 0, x.st,
                                     eu(r), nullptr, -1.f, slot_q(nt), nvec)));
                SA_AUX(x.tr, SA_CUDA(launch_pdl(k_vmul, dim3(egrid), dim3(eb), 0, x.st,
                                     ev(r), vb(r), 1.f, slot_k(nt), nvec)));
                rq[nt] = vec(slot_q(nt), vs); rk[nt] = vec(slot_k(nt), vs);
            }
            ++nt;
        }
    }
    // dQ (query sweep) and dK (key sweep).  A sweep takes at most MAXT terms;
    // longer tails (R > MAXT / 2) run one sweep per block of MAXT terms (the
    // first block carrying G), summed in fp32 in the workspace and rounded once.
    // The first block takes the remainder of 2R over MAXT, so that it carries G
    // and the full blocks follow it.
    const int nblk_t = std::max(1, (nt + simt::MAXT - 1) / simt::MAXT);
    const int first = (nt % simt::MAXT) ? nt % simt::MAXT : std::min(nt, simt::MAXT);
    // On the tensor cores a first block of at most four terms adds its modifier
    // to G inside the contraction: its K16 operands, per side (rows of the query
    // sweep and columns of the key sweep come from rq; the others from rk).
    __nv_bfloat16* augs[4] = {nullptr, nullptr, nullptr, nullptr};  // row q, col k, row k, col q
    if (std::is_same<T, __nv_bfloat16>::value && !x.p->dustbin && !direct && first > 0 &&
        first <= 4) {
        const size_t one = align_up((size_t)d.BH * d.L * 16 * 2);
        const long long n = (long long)d.BH * d.L;
        AugTerms tm;
        for (int k = 0; k < 4; ++k) {
            tm.q[k] = k < first ? rq[k] : Vec{nullptr, 0};
            tm.k[k] = k < first ? rk[k] : Vec{nullptr, 0};
        }
        tm.n = first;
        for (int i = 0; i < 4; ++i) tm.out[i] = augs[i] = (__nv_bfloat16*)(ws + l.aug + i * one);
        SA_AUX(x.tr, SA_CUDA(launch_pdl(k_aug, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, x.st, tm, d.L, d.BH)));
    }
    for (int side = 0; side < 2; ++side) {
        for (int tb = 0; tb < nblk_t; ++tb) {
            const int k0 = tb == 0 ? 0 : first + (tb - 1) * simt::MAXT;
            const int kn = tb == 0 ? first : simt::MAXT;
            simt::SweepArgs a = base_args(x);
            a.mask = mask;
            a.dust_cta = 0;
            a.nterms = kn;
            if (nblk_t > 1) {
                a.acc = (float*)(ws + l.acc);
                a.acc_in = tb > 0;
                a.acc_out = tb + 1 < nblk_t;
                a.g_off = tb > 0;
            }
            if (tb == 0) {
                a.aug_row = augs[side == 0 ? 0 : 2];
                a.aug_col = augs[side == 0 ? 1 : 3];
            }
            if (side == 0) {
                a.A = q; a.Bo = k; a.A2 = dO; a.B2 = v; a.X = k;
                a.rd = uR; a.cd = vR;
                a.cdw = x.wrow(2 * R + 1);
                a.out_mat = dq;
                for (int t = 0; t < kn; ++t) {
                    a.rv[t] = rq[k0 + t]; a.cv[t] = rk[k0 + t];
                    a.er[t] = eq[k0 + t]; a.ec[t] = ek[k0 + t]; a.cr[t] = cq[k0 + t]; a.cc[t] = ck[k0 + t];
                    a.gk[t] = gk[k0 + t];
                }
            } else {
                a.A = k; a.Bo = q; a.A2 = v; a.B2 = dO; a.X = q;
                a.rd = vR; a.cd = uR;
                a.cdw = x.wrow(2 * R);
                a.out_mat = dk;
                for (int t = 0; t < kn; ++t) {
                    a.rv[t] = rk[k0 + t]; a.cv[t] = rq[k0 + t];
                    a.er[t] = ek[k0 + t]; a.ec[t] = eq[k0 + t]; a.cr[t] = ck[k0 + t]; a.cc[t] = cq[k0 + t];
                    a.gk[t] = gk[k0 + t];
                }
            }
            if (direct && R > 0) SA_CUDA((launch_sweep<T, simt::DSD>(a, d.BH, x.st, x.tr, x.status)));
            else SA_CUDA((launch_sweep<T, simt::DS1>(a, d.BH, x.st, x.tr, x.status)));
        }
    }
    if (x.p->dustbin && dv_dust) {
        SA_AUX(x.tr, k_dvd_reduce<<<(d.H * kD + 255) / 256, 256, 0, x.st>>>(dvd, d.B, d.H,
                                                                            dv_dust));
    }
    if (x.p->dustbin && d_score) {
        double* part = (double*)(ws + l.dsc);
        SA_AUX(x.tr, k_dscore<T><<<d.BH, 256, 0, x.st>>>(dO, v_dust, mask, x.state, W_(l.ubar, 0),
                                                         W_(l.vbar, 0), vstride, R, d.L, d.H,
                                                         d.ld, x.p->dustbin_score, part));
        SA_AUX(x.tr, k_sum_parts<<<1, 256, 0, x.st>>>(part, d.BH, d_score));
    }
    return SA_OK;
}

template <typename T>
cudaError_t scan_finite(const T* x, long long n, int* status, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    long long blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    k_finite<T><<<(unsigned)blocks, 256, 0, st>>>(x, n, status);
    return cudaGetLastError();
}

}  // namespace
}  // namespace sa

using namespace sa;

extern "C" {

sa_status sinkhorn_attn_state_size(const sa_params* p, size_t* n_floats) {
    Dims d;
    sa_status s = check_params(p, &d);
    if (s != SA_OK) return s;
    if (!n_floats) return SA_ERR_INVALID_ARG;
    *n_floats = (size_t)d.BH * (2 * d.R + 2) * d.ld;
    return SA_OK;
}

sa_status sinkhorn_attn_workspace_size(const sa_params* p, size_t* fwd_bytes, size_t* bwd_bytes) {
    Dims d;
    sa_status s = check_params(p, &d);
    if (s != SA_OK) return s;
    if (fwd_bytes) *fwd_bytes = fwd_layout(d, p).total;
    if (bwd_bytes) *bwd_bytes = bwd_layout(d, p).total;
    return SA_OK;
}

}  // extern "C"

namespace {
// A shard description a sharded call can use (see sa_shard).
sa_status check_shard(const sa_params* p, const sa_shard* sh) {
    if (!sh || !sh->exchange) return SA_ERR_INVALID_ARG;
    if (sh->halo_lo < 0 || sh->halo_hi < 0 || (long long)sh->halo_lo + sh->halo_hi > p->L)
        return SA_ERR_INVALID_ARG;
    if (p->dustbin) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

sa_status fwd_call(const sa_params* p, const sa_shard* shard, const void* q, const void* k,
                   const void* v, const uint8_t* mask, const float* v_dust, void* o, float* state,
                   void* ws, size_t ws_bytes, void* stream) {
    Dims d;
    sa_status s = check_params(p, &d);
    if (s != SA_OK) return s;
    if (p->T + p->R < 1) return SA_ERR_INVALID_ARG;  // the solve needs an iteration
    if (ws_bytes < fwd_layout(d, p).total) return SA_ERR_WORKSPACE;
    if (d.BH == 0 || d.L == 0) return SA_OK;
    if (!device_ok(q) || !device_ok(k) || !device_ok(v) || !device_ok(o) || !device_ok(state) ||
        !device_ok(ws) || !mask_ok(mask))
        return SA_ERR_INVALID_ARG;
    if (p->dustbin && v_dust && !device_ok(v_dust)) return SA_ERR_INVALID_ARG;
    Ctx x;
    x.p = p;
    x.d = d;
    x.st = (cudaStream_t)stream;
    x.c = 1.0f / (std::sqrt((float)p->d) * p->eps);
    x.sst = (long long)(2 * d.R + 2) * d.ld;
    x.state = state;
    x.status = (int*)ws;
    x.tr.p = p;
    x.tr.st = x.st;
    x.shard = shard;
    if (uses_work_state(p)) x.set_work((char*)ws + fwd_layout(d, p).work);
    const float* vd = p->dustbin ? v_dust : nullptr;
    if (p->dtype == SA_F32)
        s = fwd_impl<float>(x, (const float*)q, (const float*)k, (const float*)v, mask, vd,
                            (float*)o, state);
    else
        s = fwd_impl<__nv_bfloat16>(x, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                    (const __nv_bfloat16*)v, mask, vd, (__nv_bfloat16*)o, state);
    if (s != SA_OK) return s;
    if (p->check_finite) {
        int* status = (int*)ws;
        const long long n = (long long)d.BH * d.L * kD;
        if (scan_finite<float>(state, (long long)d.BH * (2 * d.R + 2) * d.ld, status, x.st) !=
            cudaSuccess)
            return SA_ERR_CUDA;
        cudaError_t e = p->dtype == SA_F32
                            ? scan_finite<float>((const float*)o, n, status, x.st)
                            : scan_finite<__nv_bfloat16>((const __nv_bfloat16*)o, n, status, x.st);
        if (e != cudaSuccess) return SA_ERR_CUDA;
    }
    return SA_OK;
}

sa_status bwd_call(const sa_params* p, const sa_shard* shard, const void* q, const void* k,
                   const void* v, const uint8_t* mask, const float* v_dust, const void* o,
                   const void* dO, const float* state, void* dq, void* dk, void* dv,
                   float* dv_dust, float* d_dust_score, void* ws, size_t ws_bytes, void* stream) {
    Dims d;
    sa_status s = check_params(p, &d);
    if (s != SA_OK) return s;
    if (ws_bytes < bwd_layout(d, p).total) return SA_ERR_WORKSPACE;
    if (d.BH == 0 || d.L == 0) return SA_OK;
    if (!device_ok(q) || !device_ok(k) || !device_ok(v) || !device_ok(o) || !device_ok(dO) ||
        !device_ok(state) || !device_ok(dq) || !device_ok(dk) || !device_ok(dv) ||
        !device_ok(ws) || !mask_ok(mask))
        return SA_ERR_INVALID_ARG;
    if (p->dustbin && v_dust && !device_ok(v_dust)) return SA_ERR_INVALID_ARG;
    if (p->dustbin && dv_dust && !device_ok(dv_dust)) return SA_ERR_INVALID_ARG;
    if (p->dustbin && d_dust_score && !device_f32_ok(d_dust_score)) return SA_ERR_INVALID_ARG;
    Ctx x;
    x.p = p;
    x.d = d;
    x.st = (cudaStream_t)stream;
    x.c = 1.0f / (std::sqrt((float)p->d) * p->eps);
    x.sst = (long long)(2 * d.R + 2) * d.ld;
    x.state = state;
    x.status = (int*)ws;
    x.tr.p = p;
    x.tr.st = x.st;
    x.shard = shard;
    if (uses_work_state(p)) x.set_work((char*)ws + bwd_layout(d, p).work);
    const float* vd = p->dustbin ? v_dust : nullptr;
    float* dvd = p->dustbin ? dv_dust : nullptr;
    float* dsc = p->dustbin ? d_dust_score : nullptr;
    if (p->dtype == SA_F32)
        s = bwd_impl<float>(x, (const float*)q, (const float*)k, (const float*)v, mask, vd,
                            (const float*)o, (const float*)dO, (float*)dq, (float*)dk, (float*)dv,
                            dvd, dsc, (char*)ws);
    else
        s = bwd_impl<__nv_bfloat16>(
            x, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, mask, vd,
            (const __nv_bfloat16*)o, (const __nv_bfloat16*)dO, (__nv_bfloat16*)dq,
            (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, dvd, dsc, (char*)ws);
    if (s != SA_OK) return s;
    if (p->check_finite) {
        int* status = (int*)ws;
        const long long n = (long long)d.BH * d.L * kD;
        for (const void* t : {(const void*)dq, (const void*)dk, (const void*)dv}) {
            cudaError_t e =
                p->dtype == SA_F32
                    ? scan_finite<float>((const float*)t, n, status, x.st)
                    : scan_finite<__nv_bfloat16>((const __nv_bfloat16*)t, n, status, x.st);
            if (e != cudaSuccess) return SA_ERR_CUDA;
        }
    }
    return SA_OK;
}
}  // namespace

extern "C" {

sa_status sinkhorn_attn_fwd(const sa_params* p, const void* q, const void* k, const void* v,
                            const uint8_t* mask, const float* v_dust, void* o, float* state,
                            void* ws, size_t ws_bytes, void* stream) {
    return fwd_call(p, nullptr, q, k, v, mask, v_dust, o, state, ws, ws_bytes, stream);
}

sa_status sinkhorn_attn_bwd(const sa_params* p, const void* q, const void* k, const void* v,
                            const uint8_t* mask, const float* v_dust, const void* o,
                            const void* dO, const float* state, void* dq, void* dk, void* dv,
                            float* dv_dust, float* d_dust_score, void* ws, size_t ws_bytes,
                            void* stream) {
    return bwd_call(p, nullptr, q, k, v, mask, v_dust, o, dO, state, dq, dk, dv, dv_dust,
                    d_dust_score, ws, ws_bytes, stream);
}

sa_status sinkhorn_attn_fwd_sharded(const sa_params* p, const sa_shard* shard, const void* q,
                                    const void* k, const void* v, const uint8_t* mask, void* o,
                                    float* state, void* ws, size_t ws_bytes, void* stream) {
    if (!p) return SA_ERR_INVALID_ARG;
    const sa_status s = check_shard(p, shard);
    if (s != SA_OK) return s;
    return fwd_call(p, shard, q, k, v, mask, nullptr, o, state, ws, ws_bytes, stream);
}

sa_status sinkhorn_attn_bwd_sharded(const sa_params* p, const sa_shard* shard, const void* q,
                                    const void* k, const void* v, const uint8_t* mask,
                                    const void* o, const void* dO, const float* state, void* dq,
                                    void* dk, void* dv, void* ws, size_t ws_bytes, void* stream) {
    if (!p) return SA_ERR_INVALID_ARG;
    const sa_status s = check_shard(p, shard);
    if (s != SA_OK) return s;
    return bwd_call(p, shard, q, k, v, mask, nullptr, o, dO, state, dq, dk, dv, nullptr, nullptr,
                    ws, ws_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// One step with host-memory inputs and results, pipelined over problem groups
// ---------------------------------------------------------------------------
namespace {

struct Group {
    int b0, nb, h0, nh;  // batches [b0, b0 + nb), heads [h0, h0 + nh)
};

// Boundaries of n items in `parts` runs; with three or more runs the first and
// last are half as large as the others (the pipeline fills with the first
// group's copies and drains with the last one's), every run at least one item.
std::vector<int> split_runs(int n, int parts) {
    parts = std::max(1, std::min(parts, n));
    std::vector<int> cut(parts + 1, 0);
    const double total = parts >= 3 ? parts - 1.0 : parts;
    double acc = 0.0;
    for (int i = 0; i < parts; ++i) {
        acc += (parts >= 3 && (i == 0 || i == parts - 1)) ? 0.5 : 1.0;
        cut[i + 1] = (int)std::lround(acc / total * n);
    }
    cut[parts] = n;
    for (int i = 1; i <= parts; ++i) cut[i] = std::max(cut[i], cut[i - 1] + 1);  // non-empty
    for (int i = parts - 1; i >= 1; --i) cut[i] = std::min(cut[i], cut[i + 1] - 1);
    return cut;
}

// Contiguous groups of (batch, head) problems: whole batches, or runs of heads
// within each batch when there are fewer batches than groups (never with a
// dustbin, whose value and score gradients sum over every head of a batch).
std::vector<Group> plan_groups(const sa_params* p, int groups) {
    std::vector<Group> g;
    const int B = p->B, H = p->H;
    if (B <= 0 || H <= 0) return g;
    if (groups <= B || p->dustbin || H == 1) {
        const std::vector<int> cut = split_runs(B, groups);
        for (size_t i = 0; i + 1 < cut.size(); ++i) g.push_back({cut[i], cut[i + 1] - cut[i], 0, H});
    } else {
        const int per = std::min(H, (groups + B - 1) / B);
        const std::vector<int> cut = split_runs(H, per);
        for (int b = 0; b < B; ++b)
            for (size_t i = 0; i + 1 < cut.size(); ++i) g.push_back({b, 1, cut[i], cut[i + 1] - cut[i]});
    }
    return g;
}

sa_params group_params(const sa_params* p, const Group& g) {
    sa_params q = *p;
    q.B = g.nb;
    q.H = g.nh;
    q.trace_events = nullptr;
    q.trace_kinds = nullptr;
    q.trace_count = nullptr;
    q.trace_cap = 0;
    return q;
}

// Two slots (groups in flight), each with device copies of a group's inputs,
// results, dual state and fwd/bwd workspaces; then the whole mask, v_dust and
// the dustbin gradient sums.
struct HostLayout {
    size_t mat, st, fws, bws;        // bytes of one matrix, the state, the workspaces (largest group)
    size_t slot;                     // bytes of one slot
    size_t mat_off[8], st_off, fws_off, bws_off, dvd_off, dsc_off;  // within a slot
    size_t mask_off, vd_off, acc_dvd_off, acc_dsc_off, total;
};

HostLayout host_layout(const sa_params* p, const std::vector<Group>& gs) {
    HostLayout l{};
    int maxp = 0;
    Group big{0, 0, 0, 0};
    for (const Group& g : gs)
        if (g.nb * g.nh > maxp) { maxp = g.nb * g.nh; big = g; }
    const size_t es = p->dtype == SA_F32 ? 4 : 2;
    const long long ld = (long long)p->L + (p->dustbin ? 1 : 0);
    l.mat = align_up((size_t)maxp * p->L * kD * es);
    l.st = align_up((size_t)maxp * (2 * p->R + 2) * ld * sizeof(float));
    if (maxp > 0) {
        const sa_params q = group_params(p, big);
        Dims d;
        check_params(&q, &d);
        l.fws = align_up(fwd_layout(d, &q).total);
        l.bws = align_up(bwd_layout(d, &q).total);
    }
    size_t o = 0;
    for (int i = 0; i < 8; ++i) { l.mat_off[i] = o; o += l.mat; }
    l.st_off = o;  o += l.st;
    l.fws_off = o; o += l.fws;
    l.bws_off = o; o += l.bws;
    l.dvd_off = o; o += align_up((size_t)p->H * kD * sizeof(float));
    l.dsc_off = o; o += 256;
    l.slot = o;
    o = 2 * l.slot;
    l.mask_off = o;    o += align_up((size_t)p->B * p->L);
    l.vd_off = o;      o += align_up((size_t)p->H * kD * sizeof(float));
    l.acc_dvd_off = o; o += align_up((size_t)p->H * kD * sizeof(float));
    l.acc_dsc_off = o; o += 256;
    l.total = o;
    return l;
}

// Host memory, page-locked or pageable (not device memory).
bool host_ok(const void* x) {
    if (!x) return false;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, x) != cudaSuccess) {
        cudaGetLastError();
        return true;  // unknown to CUDA: pageable host memory
    }
    return at.type == cudaMemoryTypeHost || at.type == cudaMemoryTypeUnregistered;
}

// The library's two copy streams on the current device (created on first use).
sa_status copy_streams(cudaStream_t* h2d, cudaStream_t* d2h) {
    static cudaStream_t s_h2d[kMaxDevicesHS], s_d2h[kMaxDevicesHS];
    static std::mutex mu;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevicesHS) return SA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (!s_h2d[dev]) {
        if (cudaStreamCreateWithFlags(&s_h2d[dev], cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&s_d2h[dev], cudaStreamNonBlocking) != cudaSuccess)
            return SA_ERR_CUDA;
    }
    *h2d = s_h2d[dev];
    *d2h = s_d2h[dev];
    return SA_OK;
}

}  // namespace

extern "C" {

sa_status sinkhorn_attn_step_host_workspace_size(const sa_params* p, int groups, size_t* bytes) {
    Dims d;
    sa_status s = check_params(p, &d);
    if (s != SA_OK) return s;
    if (groups < 1 || !bytes) return SA_ERR_INVALID_ARG;
    *bytes = host_layout(p, plan_groups(p, groups)).total;
    return SA_OK;
}

sa_status sinkhorn_attn_step_host(const sa_params* p, const sa_host_step* io, void* ws,
                                  size_t ws_bytes, void* stream) {
    Dims d;
    sa_status s = check_params(p, &d);
    if (s != SA_OK) return s;
    if (!io || io->groups < 1) return SA_ERR_INVALID_ARG;
    if (p->check_finite) return SA_ERR_UNSUPPORTED;
    if (p->T + p->R < 1) return SA_ERR_INVALID_ARG;
    const std::vector<Group> gs = plan_groups(p, io->groups);
    const HostLayout l = host_layout(p, gs);
    if (ws_bytes < l.total) return SA_ERR_WORKSPACE;
    if (d.BH == 0 || d.L == 0) return SA_OK;
    for (const void* h : {io->q, io->k, io->v, io->dO, (const void*)io->o, (const void*)io->dq,
                          (const void*)io->dk, (const void*)io->dv})
        if (!host_ok(h)) return SA_ERR_INVALID_ARG;
    for (const void* h : {(const void*)io->mask, (const void*)io->v_dust, (const void*)io->state,
                          (const void*)io->dv_dust, (const void*)io->d_dust_score})
        if (h && !host_ok(h)) return SA_ERR_INVALID_ARG;
    if (!device_ok(ws)) return SA_ERR_INVALID_ARG;
    cudaStream_t cs = (cudaStream_t)stream, h2d = nullptr, d2h = nullptr;
    s = copy_streams(&h2d, &d2h);
    if (s != SA_OK) return s;

    char* w = (char*)ws;
    const size_t es = p->dtype == SA_F32 ? 4 : 2;
    const size_t row = (size_t)d.L * kD * es;                          // one problem's matrix
    const size_t strow = (size_t)(2 * d.R + 2) * d.ld * sizeof(float);  // one problem's state
    const bool db = p->dustbin != 0;
    uint8_t* mask_d = io->mask ? (uint8_t*)(w + l.mask_off) : nullptr;
    float* vd_d = (db && io->v_dust) ? (float*)(w + l.vd_off) : nullptr;
    float* acc_dvd = (float*)(w + l.acc_dvd_off);
    float* acc_dsc = (float*)(w + l.acc_dsc_off);

    cudaEvent_t ev_start, ev_const, ev_end, ev_in[2], ev_comp[2], ev_out[2];
    cudaEvent_t* all[] = {&ev_start, &ev_const, &ev_end, &ev_in[0], &ev_in[1],
                          &ev_comp[0], &ev_comp[1], &ev_out[0], &ev_out[1]};
    for (cudaEvent_t* e : all)
        if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return SA_ERR_CUDA;
    auto fail = [&](sa_status st) {
        for (cudaEvent_t* e : all) cudaEventDestroy(*e);
        return st;
    };
#define SA_HS(call)                                  \
    do {                                             \
        if ((call) != cudaSuccess) return fail(SA_ERR_CUDA); \
    } while (0)
    // nothing here starts before the work already queued on the caller's stream
    SA_HS(cudaEventRecord(ev_start, cs));
    SA_HS(cudaStreamWaitEvent(h2d, ev_start, 0));
    SA_HS(cudaStreamWaitEvent(d2h, ev_start, 0));
    if (mask_d) SA_HS(cudaMemcpyAsync(mask_d, io->mask, (size_t)d.B * d.L, cudaMemcpyHostToDevice, h2d));
    if (vd_d)
        SA_HS(cudaMemcpyAsync(vd_d, io->v_dust, (size_t)d.H * kD * sizeof(float),
                              cudaMemcpyHostToDevice, h2d));
    SA_HS(cudaEventRecord(ev_const, h2d));
    SA_HS(cudaStreamWaitEvent(cs, ev_const, 0));
    if (db) {
        SA_HS(cudaMemsetAsync(acc_dvd, 0, (size_t)d.H * kD * sizeof(float), cs));
        SA_HS(cudaMemsetAsync(acc_dsc, 0, sizeof(float), cs));
    }
    const void* hin[4] = {io->q, io->k, io->v, io->dO};
    void* hout[4] = {io->o, io->dq, io->dk, io->dv};
    for (size_t gi = 0; gi < gs.size(); ++gi) {
        const Group& g = gs[gi];
        const int sl = (int)(gi & 1);
        char* slot = w + sl * l.slot;
        const size_t first = (size_t)g.b0 * d.H + g.h0;  // first (batch, head) problem
        const size_t np = (size_t)g.nb * g.nh;
        // inputs: after the compute of the group that used this slot before
        if (gi >= 2) SA_HS(cudaStreamWaitEvent(h2d, ev_comp[sl], 0));
        for (int t = 0; t < 4; ++t)
            SA_HS(cudaMemcpyAsync(slot + l.mat_off[t], (const char*)hin[t] + first * row, np * row,
                                  cudaMemcpyHostToDevice, h2d));
        SA_HS(cudaEventRecord(ev_in[sl], h2d));
        // compute: after the inputs, and after the previous results left this slot
        SA_HS(cudaStreamWaitEvent(cs, ev_in[sl], 0));
        if (gi >= 2) SA_HS(cudaStreamWaitEvent(cs, ev_out[sl], 0));
        const sa_params q = group_params(p, g);
        const uint8_t* mk = mask_d ? mask_d + (size_t)g.b0 * d.L : nullptr;
        const float* vd = vd_d ? vd_d + (size_t)g.h0 * kD : nullptr;
        float* st = (float*)(slot + l.st_off);
        float* dvd = (float*)(slot + l.dvd_off);
        float* dsc = (float*)(slot + l.dsc_off);
        s = fwd_call(&q, nullptr, slot + l.mat_off[0], slot + l.mat_off[1], slot + l.mat_off[2], mk,
                     vd, slot + l.mat_off[4], st, slot + l.fws_off, l.fws, cs);
        if (s != SA_OK) return fail(s);
        s = bwd_call(&q, nullptr, slot + l.mat_off[0], slot + l.mat_off[1], slot + l.mat_off[2], mk,
                     vd, slot + l.mat_off[4], slot + l.mat_off[3], st, slot + l.mat_off[5],
                     slot + l.mat_off[6], slot + l.mat_off[7], db ? dvd : nullptr,
                     db ? dsc : nullptr, slot + l.bws_off, l.bws, cs);
        if (s != SA_OK) return fail(s);
        if (db) {
            sa::k_add<<<(d.H * kD + 255) / 256, 256, 0, cs>>>(acc_dvd, dvd, d.H * kD);
            sa::k_add<<<1, 32, 0, cs>>>(acc_dsc, dsc, 1);
            SA_HS(cudaGetLastError());
        }
        SA_HS(cudaEventRecord(ev_comp[sl], cs));
        // results: after the compute
        SA_HS(cudaStreamWaitEvent(d2h, ev_comp[sl], 0));
        for (int t = 0; t < 4; ++t)
            SA_HS(cudaMemcpyAsync((char*)hout[t] + first * row, slot + l.mat_off[4 + t], np * row,
                                  cudaMemcpyDeviceToHost, d2h));
        if (io->state)
            SA_HS(cudaMemcpyAsync((char*)io->state + first * strow, st, np * strow,
                                  cudaMemcpyDeviceToHost, d2h));
        SA_HS(cudaEventRecord(ev_out[sl], d2h));
    }
    if (db && io->dv_dust)
        SA_HS(cudaMemcpyAsync(io->dv_dust, acc_dvd, (size_t)d.H * kD * sizeof(float),
                              cudaMemcpyDeviceToHost, cs));
    if (db && io->d_dust_score)
        SA_HS(cudaMemcpyAsync(io->d_dust_score, acc_dsc, sizeof(float), cudaMemcpyDeviceToHost, cs));
    // the caller's stream covers every copy
    SA_HS(cudaEventRecord(ev_end, d2h));
    SA_HS(cudaStreamWaitEvent(cs, ev_end, 0));
#undef SA_HS
    fail(SA_OK);  // events are released once their work completes
    return SA_OK;
}

}  // extern "C"

// Fixed scratch for sinkhorn_attn_bwd_static_ws: one array per device that
// loads the library, alive until the process exits.  Host code must not use
// this name as a pointer (it is a host-side stand-in); the device address is
// looked up with cudaGetSymbolAddress, with the device current, on every call.
// Being a static __device__ array it starts zeroed, so its status word (the
// first int) reads SA_OK until a backward records a condition in it.
static __device__ __align__(256) unsigned char g_bwd_scratch[SA_STATIC_SCRATCH_BYTES];

namespace {
// Address of the scratch array on the current device.  The lookup allocates
// nothing; it is repeated on every call rather than cached, so that it stays
// right if the caller tears down and recreates the device's context.  The first
// call on a device may load the library's module there (CUDA's lazy loading),
// which is why that first call should come before any stream capture.
sa_status bwd_scratch_current_device(void** out) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess || !ptr) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    *out = ptr;
    return SA_OK;
}
}  // namespace

extern "C" {

sa_status sinkhorn_attn_bwd_static_ws(const sa_params* p, const void* q, const void* k,
                                      const void* v, const uint8_t* mask, const float* v_dust,
                                      const void* o, const void* dO, const float* state,
                                      void* dq, void* dk, void* dv, float* dv_dust,
                                      float* d_dust_score, void* stream) {
    Dims d;
    sa_status s = check_params(p, &d);
    if (s != SA_OK) return s;
    if (p->check_finite) return SA_ERR_UNSUPPORTED;
    const size_t need = bwd_layout(d, p).total;
    if (need > (size_t)SA_STATIC_SCRATCH_BYTES) return SA_ERR_WORKSPACE;
    if (d.BH == 0 || d.L == 0) return SA_OK;
    if (!device_ok(q) || !device_ok(k) || !device_ok(v) || !device_ok(o) || !device_ok(dO) ||
        !device_ok(state) || !device_ok(dq) || !device_ok(dk) || !device_ok(dv) ||
        !mask_ok(mask))
        return SA_ERR_INVALID_ARG;
    if (p->dustbin && v_dust && !device_ok(v_dust)) return SA_ERR_INVALID_ARG;
    if (p->dustbin && dv_dust && !device_ok(dv_dust)) return SA_ERR_INVALID_ARG;
    if (p->dustbin && d_dust_score && !device_f32_ok(d_dust_score)) return SA_ERR_INVALID_ARG;
    void* ws = nullptr;
    s = bwd_scratch_current_device(&ws);
    if (s != SA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    // The status word (the only part of the scratch read before it is written)
    // is not cleared here: a timeout recorded by an earlier call stays there until
    // sinkhorn_attn_poll_static reads and resets it, as with a workspace.
    Ctx x;
    x.p = p;
    x.d = d;
    x.st = st;
    x.c = 1.0f / (std::sqrt((float)p->d) * p->eps);
    x.sst = (long long)(2 * d.R + 2) * d.ld;
    x.state = state;
    x.status = (int*)ws;
    x.tr.p = p;
    x.tr.st = st;
    if (uses_work_state(p)) x.set_work((char*)ws + bwd_layout(d, p).work);
    const float* vd = p->dustbin ? v_dust : nullptr;
    float* dvd = p->dustbin ? dv_dust : nullptr;
    float* dsc = p->dustbin ? d_dust_score : nullptr;
    if (p->dtype == SA_F32)
        return bwd_impl<float>(x, (const float*)q, (const float*)k, (const float*)v, mask, vd,
                               (const float*)o, (const float*)dO, (float*)dq, (float*)dk,
                               (float*)dv, dvd, dsc, (char*)ws);
    return bwd_impl<__nv_bfloat16>(
        x, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, mask, vd,
        (const __nv_bfloat16*)o, (const __nv_bfloat16*)dO, (__nv_bfloat16*)dq,
        (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, dvd, dsc, (char*)ws);
}

sa_status sinkhorn_attn_debug_plan(const sa_params* p, int a, int b, const void* q,
                                   const void* k, const uint8_t* mask, const float* state,
                                   float* band, float* dcol, float* drow, void* stream) {
    Dims d;
    sa_status s = check_params(p, &d);
    if (s != SA_OK) return s;
    if (a < 0 || b < 0 || a > d.R || b > d.R) return SA_ERR_INVALID_ARG;
    if (d.BH == 0 || d.L == 0) return SA_OK;
    if (!device_ok(q) || !device_ok(k) || !device_ok(state) || !device_ok(band) ||
        !mask_ok(mask))
        return SA_ERR_INVALID_ARG;
    if (p->dustbin && ((dcol && !device_ok(dcol)) || (drow && !device_ok(drow))))
        return SA_ERR_INVALID_ARG;
    const float c = 1.0f / (std::sqrt((float)p->d) * p->eps);
    const dim3 grid(d.L + (p->dustbin ? 1 : 0), d.BH);
    cudaStream_t st = (cudaStream_t)stream;
    const float sd2 = p->dustbin ? p->dustbin_score * kLog2e : 0.f;
    if (p->dtype == SA_F32)
        k_debug_plan<float><<<grid, 256, 0, st>>>((const float*)q, (const float*)k, mask, state, a,
                                                  b, d.R, d.L, d.H, p->W, d.ld, c * kLog2e,
                                                  p->dustbin, sd2, band, dcol, drow);
    else
        k_debug_plan<__nv_bfloat16><<<grid, 256, 0, st>>>(
            (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, mask, state, a, b, d.R, d.L, d.H,
            p->W, d.ld, c * kLog2e, p->dustbin, sd2, band, dcol, drow);
    return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sinkhorn_attn_poll(void* ws, void* stream) {
    if (!ws) return SA_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SA_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(ws, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
        return SA_ERR_CUDA;
    return (sa_status)h;
}

sa_status sinkhorn_attn_poll_static(void* stream) {
    void* ws = nullptr;
    const sa_status s = bwd_scratch_current_device(&ws);
    if (s != SA_OK) return s;
    return sinkhorn_attn_poll(ws, stream);
}

sa_status sinkhorn_attn_debug_timeout(void* ws, long long budget_cycles, void* stream) {
    if (!ws) {  // the static scratch's status word on the current device
        const sa_status s = bwd_scratch_current_device(&ws);
        if (s != SA_OK) return s;
    }
    if (((uintptr_t)ws & 15) || !device_ok(ws)) return SA_ERR_INVALID_ARG;
    const long long b = budget_cycles < 1 ? 1 : (budget_cycles > 100000000LL ? 100000000LL : budget_cycles);
    sa::k_stall<<<1, 32, 0, (cudaStream_t)stream>>>((int*)ws, b);
    return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sinkhorn_attn_debug_exp2(const float* x, long long n, float* y_poly, float* y_mufu,
                                   void* stream) {
    if (n < 0) return SA_ERR_INVALID_ARG;
    if (n == 0) return SA_OK;
    if (!sa::device_f32_ok(x) || !sa::device_f32_ok(y_poly) || !sa::device_f32_ok(y_mufu))
        return SA_ERR_INVALID_ARG;
    const long long pairs = (n + 1) / 2;
    sa::k_exp2_pair<<<(unsigned)((pairs + 255) / 256), 256, 0, (cudaStream_t)stream>>>(x, n, y_poly,
                                                                                      y_mufu);
    return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sinkhorn_attn_sq_dist(const void* x, const void* y, long long n, sa_dtype dtype,
                               double* out, void* stream) {
    if (n < 0 || (dtype != SA_F32 && dtype != SA_BF16)) return SA_ERR_INVALID_ARG;
    if (!sa::device_ok(out) || (n > 0 && (!sa::device_ok(x) || !sa::device_ok(y))))
        return SA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(out, 0, 2 * sizeof(double), st) != cudaSuccess) return SA_ERR_CUDA;
    if (n == 0) return SA_OK;
    const long long blocks = std::min<long long>((n + 255) / 256, 148LL * 8);
    if (dtype == SA_F32)
        sa::k_sq_dist<float><<<(unsigned)blocks, 256, 0, st>>>((const float*)x, (const float*)y, n, out);
    else
        sa::k_sq_dist<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
            (const __nv_bfloat16*)x, (const __nv_bfloat16*)y, n, out);
    return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sinkhorn_attn_bias_certificate(int n_depths, const int* depths, int n_tensors,
                                         const double* sums, double tau, double* eta,
                                         int* r_star) {
    if (n_depths < 1 || n_tensors < 1 || !depths || !sums || !eta || !r_star || !(tau >= 0.0))
        return SA_ERR_INVALID_ARG;
    for (int i = 0; i < n_depths; ++i)
        if (depths[i] < 0) return SA_ERR_INVALID_ARG;
    *r_star = -1;
    for (int i = 0; i < n_depths; ++i) {
        double num = 0.0, den = 0.0;  // ||g_R - g_full||^2 and ||g_full||^2 over the tensors
        for (int t = 0; t < n_tensors; ++t) {
            const double d2 = sums[((size_t)i * n_tensors + t) * 2];
            const double n2 = sums[((size_t)i * n_tensors + t) * 2 + 1];
            if (!(d2 >= 0.0) || !(n2 >= 0.0)) return SA_ERR_INVALID_ARG;
            num += d2;
            den += n2;
        }
        eta[i] = den > 0.0 ? std::sqrt(num / den) : std::sqrt(num);
        if (eta[i] <= tau && (*r_star < 0 || depths[i] < *r_star)) *r_star = depths[i];
    }
    return SA_OK;
}

const char* sinkhorn_attn_strerror(sa_status s) {
    switch (s) {
        case SA_OK: return "success";
        case SA_ERR_INVALID_ARG: return "invalid argument (null/misaligned pointer, bad size or parameter)";
        case SA_ERR_UNSUPPORTED: return "unsupported configuration for this build";
        case SA_ERR_WORKSPACE: return "workspace too small";
        case SA_ERR_CUDA: return "CUDA runtime or launch error";
        case SA_ERR_NONFINITE: return "non-finite value in duals or outputs";
        case SA_ERR_TIMEOUT: return "bounded device wait gave up";
        case SA_ERR_EXCHANGE: return "halo exchange callback failed (sequence-sharded call)";
        case SA_ERR_BOUNDS: return "device-side bounds check failed (debug build)";
    }
    return "unknown status";
}

}  // extern "C"
