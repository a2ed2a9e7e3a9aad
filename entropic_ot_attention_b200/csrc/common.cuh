// Shared definitions of libeot: pass parameters, workspace layout, small device helpers.
//
// Method: "Blockwise Differentiable Sinkhorn Attention", technical summary (gist.science
// 2605.08123), §2.1-§2.3.  Every band sweep below evaluates, for each "row" r of one
// (batch, head) unit and the columns c in its band |r - c| <= h (h = W / 2), the score
// S_rc = scale <X_r, Y_c>.  A row half-step uses (X, Y) = (Q, K); a column half-step is the
// same sweep with (X, Y) = (K, Q) because the band and the dustbin links are symmetric.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/eot.h"

namespace eot {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxBandCtas = 1024;   // CTAs of a fused half-step launch (one per SM)
constexpr int kMaxR = 8;
constexpr int kMaxMods = 2 * kMaxR;

// Device status bits (first word of every workspace).
constexpr uint32_t kStatusNonFinite = 1u;
constexpr uint32_t kStatusTimeout = 2u;

// Problem geometry as the kernels see it.
struct Geom {
    int B, H, BH, L, d;
    int h;          // band half-width W / 2
    int D;          // dustbin position, or -1 (active iff logm[D] > -inf)
    int dself;      // (D, D) in the support
    float scale;    // score scale (natural units)
    int dtype;      // eot_dtype
};

// One log-sum-exp half-step (§2.1):
//   out_r = logm_r - LSE_{c in band(r), active, c != D} (S_rc + colpot_c) [+ dustbin entry]
struct LsePass {
    Geom g;
    const void* X;          // [BH, L, d] row-side operand of S
    const void* Y;          // [BH, L, d] column-side operand of S
    const float* logm;      // [B, L] log marginals, -inf for inactive positions
    const float* colpot;    // potential of the column side (natural log)
    const float* stab;      // previous value of this row potential, or nullptr
    float* out;             // new row potential (0 for inactive rows)
    size_t pstride;         // unit stride of colpot / stab / out (elements): L or (R+1) L
    const float* colbias2;  // [BH, L] log2(e) * colpot, -inf for inactive columns and the dustbin
    float* out_bias2;       // [BH, L] same masking of the new potential (for the next half-step)
    const uint32_t* tile_bits;  // [B][tile_words(L)]: 128-position tiles holding an active non-dustbin token
    const float* sd_term;   // [BH, L] S between row r and the dustbin column (dustbin only)
    const float* sd_dense;  // [BH, L] S between the dustbin row and column c (dustbin only)
    float* dpart;           // dense dustbin row: per-CTA partial sums (dustbin only)
    uint32_t* dcnt;         // [BH] CTAs of the dense dustbin row done (zero between launches)
    uint32_t* status;
    // tensor-core kernels: also write each output position's column-bias operand row here
    // ([BH L, 16] bf16; read by the fused half-steps that follow), or nullptr
    __nv_bfloat16* ext_out;
    // tensor-core kernels: the CTAs' item ranges (launch_schedule), or nullptr for equal ranges
    const int* bounds;
};

// One backward sweep (§2.2).  With Pt_rc = exp(S_rc + pr_r + pc_c) on the support:
//   scalar : sout_r = f_r * ( sum_c Pt_rc * dP_rc [if s_dp] + hv_r * sum_c Pt_rc * m_c )
//   vector : vout_r = vscale * sum_c coef_rc Z_c,
//            coef_rc = Pt_rc * ( (v_dp ? dP_rc : 1) - sum_k xr_k[r] * yc_k[c] )
// where dP_rc = <A_r, Bm_c>.  Any of the vectors may be nullptr when unused.
struct BwdPass {
    Geom g;
    const void* X;
    const void* Y;
    const void* A;          // row-side dP operand
    const void* Bm;         // column-side dP operand
    const void* Z;          // column-side operand of the vector output
    const float* logm;
    const float* pr;        // [BH, L]
    const float* pc;        // [BH, L] (value at D used for the dustbin links)
    const float* pcm2;      // [BH, L] log2(e) * pc, -inf for inactive columns and the dustbin
    float* sout;            // scalar output or nullptr
    const float* f;
    const float* hv;
    const float* m;
    int s_dp;
    void* vout;             // vector output [BH, L, d] (dtype) or nullptr
    float vscale;
    int v_dp;
    int nmod;
    const float* xr[kMaxMods];
    const float* yc[kMaxMods];
    const float* sd_term;   // dustbin links of S (as in LsePass)
    const float* sd_dense;
    const float* dp_term;   // <A_r, Bm_D>
    const float* dp_dense;  // <A_D, Bm_c>
    const float* zero_vec;  // [BH, L] zeros (padding of the modifier list), or nullptr
    __nv_bfloat16* pcache;  // row sweep (alpha_R): cache its plan tiles here (tensor-core kernels), or nullptr
    // Column sweep beta_R (tensor-core kernels): also write, per column position c, partial sums
    // of Pt_rc dP_rc over the 32 rows r of each (row tile, TMEM lane quadrant q) into
    // s1part[(o * 4 + q) s1stride + bh L + c], o = column tile - row tile + s1E; or nullptr.
    float* s1part;
    size_t s1stride;
    int s1E;
    const float* sadd;      // staircase-form sweeps: out_r = f_r (hv_r sum_c ... + sadd_r), or nullptr
    // staircase-form sweeps on the tensor cores (d = 128, W >= 512): the column-bias operand rows
    // of this pass's column bias pcm2 ([BH L, 16] bf16, see band_ext_row), or nullptr
    const __nv_bfloat16* cext;
    // dQ / dK (tensor-core kernels, no dustbin): the modifiers as [BH L, 16] bf16 operand rows
    // (xext row side, yext column side; see BwdVecArgs) to fold into the dP product, or nullptr
    const __nv_bfloat16* xext;
    const __nv_bfloat16* yext;
    const uint32_t* tile_bits;  // as in LsePass (tensor-core staircase sums)
    const int* bounds;          // as in LsePass (tensor-core staircase sums)
    // tensor-core sweeps: the row-tile jobs in the order the persistent CTAs take them by stride
    // (launch_schedule: the active ones first), or nullptr for the natural order
    const int* jobs;
    float* dpart;           // as in LsePass
    uint32_t* dcnt;
    uint32_t* status;
};

// Workspace layout.  Every region is 256-byte aligned; offsets in bytes.
struct WsLayout {
    size_t status, logm, sd_row, sd_col, e1, e2;
    size_t dpart, dcnt;     // dense dustbin row: per-CTA partials and completion counters
    size_t opr, opc, opcm;  // forward output pass: row / column biases
    size_t ub2, vb2;        // forward: masked log2 potentials feeding the next half-step
    size_t gbar;            // forward: grid-barrier counters of the fused half-steps [2 (T + R)]
    size_t bounds;          // item ranges of the band kernel's CTAs [kMaxBandCtas + 1]
    size_t jobs;            // job order of the sweep kernel [BH L / 128]
    size_t part;            // forward, one exponential per iteration: column partial sums [BH][L/128][window][128]
    size_t tbits;           // active-tile bitmask [B][tile_words(L)]
    size_t pcm;             // backward: masked log2 column bias
    size_t zero;            // backward: a vector of zeros
    size_t pr, pc, f, hv, m;
    size_t xr, yc;          // kMaxMods vectors each, [BH, L]
    size_t alpha, beta;     // (R + 1) vectors each, [BH, L]
    size_t pcache;          // backward with the cached reference plan: bf16 band store [BH, L, 2 h + 128]
    size_t s1part, sadd;    // backward, split alpha_R sweep: partial sums [4 (2 E + 1)][BH, L] and their total
    bool s1split;
    size_t xext, yext;      // backward, folded modifiers: [BH L, 16] bf16 each
    bool fold;
    size_t ue, ve;          // forward, fused d = 128 half-steps: column-bias operand rows [BH L, 16] bf16 of u and v
    bool bext;
    size_t cext;            // backward, band sums of wide d = 128 bands: column-bias operand rows [BH L, 16] bf16
    bool bcext;
    size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
// The dense dustbin row is split over CTAs of kDCols columns (plus the (D, D) entry).
constexpr int kDCols = 256;
__host__ __device__ inline int dustbin_splits(int L) { return (L + 1 + kDCols - 1) / kDCols; }
__host__ __device__ inline int tile_words(int L) { return (L / 128 + 31) / 32; }

// Window of a 128-row strip: the 128-column tiles that meet the band of its rows,
// [128 s - h, 128 s + 127 + h]; the most any strip has (L / 128 at most).
inline int iter_window_tiles(int L, int h) {
    const long n = 1L + (long(h) + 127) / 128 + (long(h) + 127) / 128;
    return int(n < L / 128 ? n : L / 128);
}
// Problems the one-exponential-per-iteration forward can run (tensor cores, bf16, no dustbin, a
// stopped base, a window of at most nine tiles); they get its column-partial workspace.
inline bool iter_schedule_possible(const eot_problem& p) {
    return p.dtype == EOT_BF16 && (p.d == 64 || p.d == 128) && !p.dustbin && p.T >= 1 && p.impl != EOT_IMPL_SIMT &&
           p.L >= 128 && iter_window_tiles(p.L, p.W / 2) <= 9;
}

// The backward caches its reference plan (a bf16 band store of 2 h + 128 entries a row) only
// when asked to (eot_set_backward_schedule) and for tensor-core problems without a dustbin whose
// half-width h is a multiple of 128 and whose tail has a staircase (R >= 2).
int backward_schedule();
inline bool cache_plan_possible(const eot_problem& p) {
    return backward_schedule() == 1 && p.dtype == EOT_BF16 && (p.d == 64 || p.d == 128) && !p.dustbin &&
           p.impl != EOT_IMPL_SIMT && (p.W / 2) % 128 == 0 && p.R >= 2;
}

// The alpha_R sweep of the backward is split (the column sweep beta_R also writes the partial row
// sums of Pt dP, and alpha_R becomes a staircase-form band sum) for tensor-core problems without
// a dustbin whose band reaches at most E = ceil(h / 128) <= 7 tiles to each side, unless the
// cached-plan schedule is selected (its alpha_R sweep stores the plan).
inline int s1_reach(int W) { return (W / 2 + 127) / 128; }
inline bool s1_split_possible(const eot_problem& p) {
    return p.dtype == EOT_BF16 && (p.d == 64 || p.d == 128) && !p.dustbin && p.impl != EOT_IMPL_SIMT && p.R >= 1 &&
           p.L % 128 == 0 && s1_reach(p.W) <= 7 && !cache_plan_possible(p);
}
inline size_t s1_slots(int W) { return size_t(4) * size_t(2 * s1_reach(W) + 1); }

// The rank-2R modifier term of the dQ / dK sweeps is folded into their dP product (three bf16
// products per modifier, hi x hi + hi x lo + lo x hi, in one K = 16 step) for tensor-core
// problems without a dustbin and with 2 R <= kMaxFoldMods.
constexpr int kMaxFoldMods = 5;
inline bool fold_possible(const eot_problem& p) {
    return p.dtype == EOT_BF16 && (p.d == 64 || p.d == 128) && !p.dustbin && p.impl != EOT_IMPL_SIMT && p.R >= 1 &&
           2 * p.R <= kMaxFoldMods && p.L % 128 == 0;
}

inline WsLayout ws_layout(const eot_problem& p, bool bwd) {
    WsLayout w{};
    const size_t BH = size_t(p.B) * p.H, L = size_t(p.L);
    const size_t vec = align256(BH * L * sizeof(float));
    size_t o = 0;
    w.status = o; o += 256;
    w.logm = o; o += align256(size_t(p.B) * L * sizeof(float));
    if (p.dustbin) {
        w.sd_row = o; o += vec;
        w.sd_col = o; o += vec;
        if (bwd) { w.e1 = o; o += vec; w.e2 = o; o += vec; }
        w.dpart = o; o += align256(BH * size_t(dustbin_splits(p.L)) * size_t(p.d + 2) * sizeof(float));
        w.dcnt = o; o += align256(BH * sizeof(uint32_t));
    }
    if (!bwd) {
        w.opr = o; o += vec;
        w.opc = o; o += vec;
        w.opcm = o; o += vec;
        w.ub2 = o; o += vec;
        w.vb2 = o; o += vec;
        w.gbar = o; o += align256(size_t(2) * (size_t(p.T) + size_t(p.R)) * sizeof(uint32_t) + 4);
        if (p.dtype == EOT_BF16 && p.d == 128 && p.impl != EOT_IMPL_SIMT && p.L % 128 == 0 && p.W / 2 >= 256) {
            w.bext = true;
            w.ue = o; o += align256(BH * L * 32);
            w.ve = o; o += align256(BH * L * 32);
        }
        if (iter_schedule_possible(p)) {
            w.part = o;
            o += align256(BH * size_t(p.L / 128) * size_t(iter_window_tiles(p.L, p.W / 2)) * 128 * sizeof(float));
        }
    }
    w.tbits = o; o += align256(size_t(p.B) * size_t((p.L / 128 + 31) / 32) * 4);
    w.bounds = o; o += align256(size_t(kMaxBandCtas + 1) * sizeof(int));
    w.jobs = o; o += align256(BH * size_t(p.L / 128) * sizeof(int));
    if (bwd) {
        w.pr = o; o += vec;
        w.pc = o; o += vec;
        w.f = o; o += vec;
        w.hv = o; o += vec;
        w.m = o; o += vec;
        w.pcm = o; o += vec;
        w.zero = o; o += vec;
        w.xr = o; o += vec * 2 * p.R;
        w.yc = o; o += vec * 2 * p.R;
        w.alpha = o; o += vec * (p.R + 1);
        w.beta = o; o += vec * (p.R + 1);
        if (cache_plan_possible(p)) {
            w.pcache = o;
            o += align256(BH * L * size_t(p.W / 2 * 2 + 128) * 2);
        }
        if (s1_split_possible(p)) {
            w.s1split = true;
            w.s1part = o; o += s1_slots(p.W) * vec;
            w.sadd = o; o += vec;
        }
        if (p.dtype == EOT_BF16 && p.d == 128 && p.impl != EOT_IMPL_SIMT && p.L % 128 == 0 && p.W / 2 >= 256) {
            w.bcext = true;
            w.cext = o; o += align256(BH * L * 32);
        }
        if (fold_possible(p)) {
            w.fold = true;
            w.xext = o; o += align256(BH * L * 32);
            w.yext = o; o += align256(BH * L * 32);
        }
    }
    w.total = o;
    return w;
}

// ---------------------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// The column bias enters the score product of the band kernel (d = 128, wide bands: fused
// half-steps and weighted band sums): one more K = 16 step
// multiplies a constant row operand (1, 1, 1, 0, ...) with a column operand row
// (y_hi, y_mid, y_lo, 0, ...) carrying y = b_c / (scale log2 e), b_c the column's masked log2
// potential, as three bf16 parts (fp32 accuracy); the accumulator then holds S + y and the
// epilogue forms the exponent with one packed FMA, acc * scale log2 e + st_r.  A column
// that never enters a band sum (inactive, the dustbin) carries y = -2^100.
__device__ __forceinline__ void band_ext_row(__nv_bfloat16* dst, float b2, float isl2) {
    const float y = b2 == neg_inf() ? -1.2676506e30f : b2 * isl2;   // isl2 = 1 / (scale log2 e); -2^100
    const __nv_bfloat16 hi = __float2bfloat16_rn(y);
    const float r1 = y - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    __nv_bfloat162 p0, p1;
    p0.x = hi;
    p0.y = mid;
    p1.x = lo;
    p1.y = __float2bfloat16_rn(0.f);
    uint4 w0;
    w0.x = *reinterpret_cast<const uint32_t*>(&p0);
    w0.y = *reinterpret_cast<const uint32_t*>(&p1);
    w0.z = 0u;
    w0.w = 0u;
    uint4* d = reinterpret_cast<uint4*>(dst);
    d[0] = w0;
    d[1] = make_uint4(0u, 0u, 0u, 0u);
}


// Merge two (max, sum) log-sum-exp partials in the log2 domain.
__device__ __forceinline__ void lse2_merge(float& m, float& s, float m2, float s2) {
    float M = fmaxf(m, m2);
    if (M == neg_inf()) return;
    float a = (m == neg_inf()) ? 0.f : s * exp2f(m - M);
    float b = (m2 == neg_inf()) ? 0.f : s2 * exp2f(m2 - M);
    m = M;
    s = a + b;
}

__device__ __forceinline__ void lse2_add(float& m, float& s, float x) {
    if (x == neg_inf()) return;
    if (x > m) {
        s = (m == neg_inf() ? 0.f : s * exp2f(m - x)) + 1.f;
        m = x;
    } else {
        s += exp2f(x - m);
    }
}

}  // namespace eot
