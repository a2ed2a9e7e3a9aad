// CUDA-core kernels of libeot: marginal/dustbin preparation, the fp32 (and reference bf16)
// band sweeps, the dense dustbin row, and the backward vector preparation.
//
// Method: "Blockwise Differentiable Sinkhorn Attention", technical summary (gist.science
// 2605.08123): §2.1 balanced log-domain Sinkhorn on a fixed band support with the
// temperature absorbed into S; §2.2 exact adjoint of the refinement tail through one
// reference plan and per-row / per-column orbit factors; §2.3 dustbin token on an extended
// state space.
//
// Tiling of the CUDA-core sweeps: a CTA owns 32 rows of one unit and walks the 32-column
// tiles that intersect the band of those rows.  Each of its 8 warps owns 4 rows; lane l
// owns column l of the current tile.  Row-side operands stay in shared memory for the
// whole sweep, column-side operands are staged per tile.  Scores are exact fp32 dot
// products (FFMA), which keeps fp32 inputs at fp32 accuracy.
#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"

namespace eot {

constexpr int kSB = 32;    // rows per CTA == columns per tile
constexpr int kSNT = 256;  // threads per CTA

// ---------------------------------------------------------------------------------------
// Preparation
// ---------------------------------------------------------------------------------------

// Uniform marginals over the active real tokens (§2.1), dustbin mass (§2.3).  One CTA per
// batch row.  logm[b, i] = log a_i, -inf for inactive positions.
// One CTA of 1024 threads per batch row (L is a multiple of 128): count the real tokens (mask
// bytes read 16 at a time when the mask is 16-byte aligned), then write the row's log marginals
// 4 at a time.
// Block (b, j): counts the active real tokens of batch row b (every block of the row reads the
// whole mask row, from L2 after the first) and writes positions [j kPrepSlice, (j + 1) kPrepSlice)
// of the log marginals and, when asked, of the tile bits (the slice is word j of the row: warp w
// votes for tile 32 j + w) and of the zero potential's masked log2 bias of every head.
constexpr int kPrepSlice = 4096;
static_assert(kPrepSlice == 32 * 128, "one 32-bit word of tile bits per slice");
__global__ void __launch_bounds__(1024) prep_marginals_kernel(Geom g, const uint8_t* mask, int dustbin,
                                                              float mass, float* logm, uint32_t* status,
                                                              uint32_t* bits, float* bias2) {
    const int b = blockIdx.x;
    const int L = g.L;
    const int w0 = blockIdx.y * kPrepSlice, w1 = min(L, w0 + kPrepSlice);
    const int D = dustbin ? g.D : L;
    const uint8_t* mrow = mask ? mask + size_t(b) * L : nullptr;
    const bool vec = mrow && (reinterpret_cast<uintptr_t>(mask) & 15) == 0;
    __shared__ int red[32];
    int cnt = 0;
    if (!mrow) {
        cnt = threadIdx.x == 0 ? min(L, D) : 0;
    } else if (vec) {
        for (int i0 = threadIdx.x * 16; i0 < L; i0 += blockDim.x * 16) {
            const uint4 w = *reinterpret_cast<const uint4*>(mrow + i0);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < 16; ++j) cnt += (((ww[j >> 2] >> (8 * (j & 3))) & 0xffu) != 0u) && (i0 + j < D);
        }
    } else {
        for (int i = threadIdx.x; i < L; i += blockDim.x) cnt += (mrow[i] != 0) && (i < D);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = cnt;
    __syncthreads();
    int n = 0;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) n += red[w];
    const bool use_db = dustbin && n > 0 && mass > 0.f;
    const double real_mass = use_db ? (1.0 - double(mass)) : 1.0;
    const float lr = n > 0 ? float(log(real_mass / double(n))) : neg_inf();
    const float ld = use_db ? float(log(double(mass))) : neg_inf();
    __shared__ uint32_t word;
    if (threadIdx.x == 0) word = 0u;
    __syncthreads();
    // one pass of 4 positions a thread covers the slice (kPrepSlice = 4 x 1024)
    const int i0 = w0 + threadIdx.x * 4;
    bool any = false;
    if (i0 < w1) {
        float v[4], bz[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j;
            const bool real = (mrow ? (mrow[i] != 0) : true) && (i < D);
            any |= real;
            v[j] = real ? lr : neg_inf();
            bz[j] = real ? 0.f : neg_inf();   // the dustbin never enters a band sum
            if (dustbin && i == D) v[j] = ld;
        }
        *reinterpret_cast<float4*>(logm + size_t(b) * L + i0) = make_float4(v[0], v[1], v[2], v[3]);
        if (bias2)
            for (int hh = 0; hh < g.H; ++hh)
                *reinterpret_cast<float4*>(bias2 + (size_t(b) * g.H + hh) * L + i0) = make_float4(bz[0], bz[1], bz[2], bz[3]);
    }
    if (bits) {
        // warp w holds the 128 positions of tile 32 j + w
        const unsigned vote = __ballot_sync(0xffffffffu, any);
        if ((threadIdx.x & 31) == 0 && vote) atomicOr(&word, 1u << (threadIdx.x >> 5));
        __syncthreads();
        if (threadIdx.x == 0) bits[size_t(b) * tile_words(L) + blockIdx.y] = word;
    }
    if (b == 0 && blockIdx.y == 0 && threadIdx.x == 0 && status) *status = 0u;
}

// Dustbin link vectors: out_term[r] = s1 * <P_r, Q_D>, out_dense[r] = s1 * <P_D, Q_r> for
// every position r of every unit (used for S and, in the backward, for dP).  One warp per row:
// lane l takes elements l, l + 32, ... (coalesced), the two dots meet by shuffles.
template <typename T>
__global__ void __launch_bounds__(256) prep_dustbin_dots_kernel(Geom g, const T* P, const T* Qm, float s1,
                                                                float* out_term, float* out_dense) {
    // 8 lanes per row, each summing its d / 8 consecutive elements (independent loads in flight),
    // then a 3-step reduction within the 8 lanes; 32 rows per block
    const int bh = blockIdx.y, sub = threadIdx.x & 7;
    const int r = blockIdx.x * (blockDim.x >> 3) + (threadIdx.x >> 3);
    const bool live = r < g.L;
    const size_t base = size_t(bh) * g.L;
    const int per = g.d >> 3, k0 = sub * per;   // d is a multiple of 8
    float a = 0.f, b = 0.f;
    if (live) {
        const T* pr = P + (base + r) * g.d + k0;
        const T* pD = P + (base + g.D) * g.d + k0;
        const T* qr = Qm + (base + r) * g.d + k0;
        const T* qD = Qm + (base + g.D) * g.d + k0;
#pragma unroll 4
        for (int k = 0; k < per; ++k) {
            a = fmaf(to_f(pr[k]), to_f(qD[k]), a);
            b = fmaf(to_f(pD[k]), to_f(qr[k]), b);
        }
    }
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, off);
        b += __shfl_xor_sync(0xffffffffu, b, off);
    }
    if (live && sub == 0) {
        out_term[base + r] = s1 * a;
        out_dense[base + r] = s1 * b;
    }
}

// ---------------------------------------------------------------------------------------
// Forward half-step on CUDA cores (online max; fp32 scores)
// ---------------------------------------------------------------------------------------
// Rows [32 rblk, 32 rblk + 32) of unit bh (the whole CTA takes part).
template <typename T>
__device__ void simt_lse_item(const LsePass& p, int rblk, int bh, float* sm) {
    const int d = p.g.d, ld = d + 1, L = p.g.L, h = p.g.h, D = p.g.D;
    float* Xs = sm;
    float* Ys = Xs + kSB * ld;
    float* bs = Ys + kSB * ld;
    const int b = bh / p.g.H;
    const int r0 = rblk * kSB;
    const size_t base = size_t(bh) * L;
    const size_t pb = size_t(bh) * p.pstride;
    const T* X = static_cast<const T*>(p.X) + base * d;
    const T* Y = static_cast<const T*>(p.Y) + base * d;
    const float* logm = p.logm + size_t(b) * L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float sl2 = p.g.scale * kLog2e;
    const bool d_act = (D >= 0) && (logm[D] != neg_inf());

    for (int e = threadIdx.x; e < kSB * d; e += kSNT) {
        int r = e / d, k = e - r * d;
        Xs[r * ld + k] = to_f(X[size_t(r0 + r) * d + k]);
    }
    float m[4], s[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) { m[q] = neg_inf(); s[q] = 0.f; }

    const int clo = max(0, r0 - h), chi = min(L - 1, r0 + kSB - 1 + h);
    for (int t = clo / kSB; t <= chi / kSB; ++t) {
        const int c0 = t * kSB;
        __syncthreads();
        for (int e = threadIdx.x; e < kSB * d; e += kSNT) {
            int r = e / d, k = e - r * d;
            Ys[r * ld + k] = to_f(Y[size_t(c0 + r) * d + k]);
        }
        if (threadIdx.x < kSB) {
            const int c = c0 + threadIdx.x;
            const bool act = logm[c] != neg_inf() && c != D;
            bs[threadIdx.x] = act ? p.colpot[pb + c] * kLog2e : neg_inf();
        }
        __syncthreads();
        const int c = c0 + lane;
        const float bc = bs[lane];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int rl = warp * 4 + q, r = r0 + rl;
            float acc = 0.f;
            for (int k = 0; k < d; ++k) acc = fmaf(Xs[rl * ld + k], Ys[lane * ld + k], acc);
            float x = fmaf(acc, sl2, bc);
            if (abs(r - c) > h) x = neg_inf();
            lse2_add(m[q], s[q], x);
        }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            float m2 = __shfl_xor_sync(0xffffffffu, m[q], off);
            float s2 = __shfl_xor_sync(0xffffffffu, s[q], off);
            lse2_merge(m[q], s[q], m2, s2);
        }
    }
    if (lane < 4) {
        const int q = lane;
        const int r = r0 + warp * 4 + q;
        float mq = m[0], sq = s[0];
#pragma unroll
        for (int j = 1; j < 4; ++j) if (q == j) { mq = m[j]; sq = s[j]; }
        const float lm = logm[r];
        if (r == D && d_act) return;  // written by the dense dustbin row
        float outv = 0.f, ob = neg_inf();
        if (lm != neg_inf()) {
            if (d_act) lse2_add(mq, sq, (p.sd_term[base + r] + p.colpot[pb + D]) * kLog2e);
            outv = lm - (mq + log2f(sq)) * kLn2;
            if (!isfinite(outv)) atomicOr(p.status, kStatusNonFinite);
            ob = outv * kLog2e;
        }
        p.out[pb + r] = outv;
        p.out_bias2[base + r] = ob;
    }
}

template <typename T>
__global__ void __launch_bounds__(kSNT) simt_lse_kernel(LsePass p) {
    extern __shared__ float sm[];
    simt_lse_item<T>(p, blockIdx.x, blockIdx.y, sm);
}

// Every half-step of a forward without a dustbin in one cooperative launch: half-step hs
// (row when even: X = Q, Y = K; column when odd: X = K, Y = Q) of iteration it = hs / 2 reads and
// writes potential slot 0 for the first T iterations and slot it - T + 1 after (the column
// potential of a row half-step comes from the previous iteration's slot); a grid-wide barrier
// (gbar[hs]: CTAs done with half-step hs) separates consecutive half-steps.
template <typename T>
__global__ void __launch_bounds__(kSNT) simt_lse_fused_kernel(LsePass row, const void* Qp, const void* Kp, float* u_tail,
                                                              float* v_tail, float* ub2, float* vb2, int nhs, int Tb,
                                                              uint32_t* gbar) {
    extern __shared__ float sm[];
    __shared__ int abort_flag;
    if (threadIdx.x == 0) abort_flag = 0;
    __syncthreads();
    const int L = row.g.L, items = (L / kSB) * row.g.BH;
    for (int hs = 0; hs < nhs; ++hs) {
        if (hs > 0) {
            // every CTA is done with half-step hs - 1
            if (threadIdx.x == 0) ptx::grid_wait(gbar + hs - 1, gridDim.x, &abort_flag, row.status);
            __syncthreads();
            if (abort_flag) return;
        }
        const int it = hs >> 1;
        const int sout = it < Tb ? 0 : it - Tb + 1, sin = it < Tb ? 0 : it - Tb;
        LsePass p = row;
        if ((hs & 1) == 0) {
            p.X = Qp;
            p.Y = Kp;
            p.colpot = v_tail + size_t(sin) * L;
            p.out = u_tail + size_t(sout) * L;
            p.out_bias2 = ub2;
        } else {
            p.X = Kp;
            p.Y = Qp;
            p.colpot = u_tail + size_t(sout) * L;
            p.out = v_tail + size_t(sout) * L;
            p.out_bias2 = vb2;
        }
        for (int item = blockIdx.x; item < items; item += gridDim.x) {
            __syncthreads();   // the previous item's tiles are no longer read
            simt_lse_item<T>(p, item % (L / kSB), item / (L / kSB), sm);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            atomicAdd(gbar + hs, 1u);
        }
    }
}

// Dense dustbin row of a half-step: out_D = logm_D - LSE_c (S_Dc + colpot_c) over every
// active real c, plus (D, D) when it is in the support.  One CTA per unit.
__global__ void __launch_bounds__(256) dustbin_lse_kernel(LsePass p) {
    // CTA (split, unit): columns [split * kDCols, ...) of the dense dustbin row (column L stands
    // for the (D, D) entry); the last CTA of a unit to finish merges the partial sums.
    const int split = blockIdx.x, ns = gridDim.x, bh = blockIdx.y, b = bh / p.g.H, L = p.g.L, D = p.g.D;
    const size_t base = size_t(bh) * L;
    const size_t pb = size_t(bh) * p.pstride;
    const float* logm = p.logm + size_t(b) * L;
    if (D < 0 || logm[D] == neg_inf()) return;
    float m = neg_inf(), s = 0.f;
    const int c_end = min(L + 1, (split + 1) * kDCols);
    for (int c = split * kDCols + threadIdx.x; c < c_end; c += blockDim.x) {
        if (c == L) {
            if (p.g.dself) lse2_add(m, s, (p.sd_term[base + D] + p.colpot[pb + D]) * kLog2e);
            continue;
        }
        if (c == D || logm[c] == neg_inf()) continue;
        lse2_add(m, s, (p.sd_dense[base + c] + p.colpot[pb + c]) * kLog2e);
    }
    __shared__ float sm_m[256], sm_s[256];
    __shared__ int last;
    sm_m[threadIdx.x] = m;
    sm_s[threadIdx.x] = s;
    __syncthreads();
    for (int st = 128; st > 0; st >>= 1) {
        if (threadIdx.x < st) {
            float a = sm_m[threadIdx.x], bb = sm_s[threadIdx.x];
            lse2_merge(a, bb, sm_m[threadIdx.x + st], sm_s[threadIdx.x + st]);
            sm_m[threadIdx.x] = a;
            sm_s[threadIdx.x] = bb;
        }
        __syncthreads();
    }
    float* part = p.dpart + size_t(bh) * ns * 2;
    if (threadIdx.x == 0) {
        part[2 * split] = sm_m[0];
        part[2 * split + 1] = sm_s[0];
        __threadfence();
        last = atomicAdd(p.dcnt + bh, 1u) == unsigned(ns - 1);
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    // the unit's partials, merged by the whole block in a fixed order (strided, then a tree)
    float mm = neg_inf(), ss = 0.f;
    for (int i = threadIdx.x; i < ns; i += blockDim.x) lse2_merge(mm, ss, __ldcg(part + 2 * i), __ldcg(part + 2 * i + 1));
    sm_m[threadIdx.x] = mm;
    sm_s[threadIdx.x] = ss;
    __syncthreads();
    for (int st = 128; st > 0; st >>= 1) {
        if (threadIdx.x < st) {
            float a = sm_m[threadIdx.x], bb = sm_s[threadIdx.x];
            lse2_merge(a, bb, sm_m[threadIdx.x + st], sm_s[threadIdx.x + st]);
            sm_m[threadIdx.x] = a;
            sm_s[threadIdx.x] = bb;
        }
        __syncthreads();
    }
    if (threadIdx.x != 0) return;
    p.dcnt[bh] = 0u;   // ready for the next launch of this call
    float outv = logm[D] - (sm_m[0] + log2f(sm_s[0])) * kLn2;
    if (!isfinite(outv)) atomicOr(p.status, kStatusNonFinite);
    p.out[pb + D] = outv;
    p.out_bias2[base + D] = neg_inf();   // the dustbin never enters a band sum
}

// ---------------------------------------------------------------------------------------
// Backward sweep on CUDA cores
// ---------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kSNT) simt_bwd_kernel(BwdPass p) {
    extern __shared__ float sm[];
    const int d = p.g.d, ld = d + 1, L = p.g.L, h = p.g.h, D = p.g.D;
    const int nm = p.nmod;
    const bool has_dp = (p.sout && p.s_dp) || (p.vout && p.v_dp);
    float* Xs = sm;                       // [32][ld]
    float* As = Xs + kSB * ld;            // [32][ld]
    float* Ys = As + kSB * ld;            // [32][ld]
    float* Bs = Ys + kSB * ld;            // [32][ld]
    float* Zs = Bs + kSB * ld;            // [32][ld]
    float* Cs = Zs + kSB * ld;            // [32][33] coefficients
    float* colv = Cs + kSB * 33;          // [2 + nm][32]: pc, m, yc...
    float* rowv = colv + (2 + kMaxMods) * kSB;  // [3 + nm][32]: pr, f, hv, xr...
    const int bh = blockIdx.y, b = bh / p.g.H;
    const int r0 = blockIdx.x * kSB;
    const size_t base = size_t(bh) * L;
    const float* logm = p.logm + size_t(b) * L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float sc = p.g.scale;
    const bool d_act = (D >= 0) && (logm[D] != neg_inf());
    const T* X = static_cast<const T*>(p.X) + base * d;
    const T* Y = static_cast<const T*>(p.Y) + base * d;
    const T* A = has_dp ? static_cast<const T*>(p.A) + base * d : nullptr;
    const T* Bm = has_dp ? static_cast<const T*>(p.Bm) + base * d : nullptr;
    const T* Z = p.vout ? static_cast<const T*>(p.Z) + base * d : nullptr;

    for (int e = threadIdx.x; e < kSB * d; e += kSNT) {
        int r = e / d, k = e - r * d;
        Xs[r * ld + k] = to_f(X[size_t(r0 + r) * d + k]);
        if (has_dp) As[r * ld + k] = to_f(A[size_t(r0 + r) * d + k]);
    }
    if (threadIdx.x < kSB) {
        const int r = r0 + threadIdx.x;
        rowv[0 * kSB + threadIdx.x] = p.pr[base + r];
        rowv[1 * kSB + threadIdx.x] = p.f ? p.f[base + r] : 1.f;
        rowv[2 * kSB + threadIdx.x] = p.hv ? p.hv[base + r] : 0.f;
        for (int k = 0; k < nm; ++k) rowv[(3 + k) * kSB + threadIdx.x] = p.xr[k][base + r];
    }
    float s1[4], s2[4], acc[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        s1[q] = s2[q] = 0.f;
#pragma unroll
        for (int z = 0; z < 4; ++z) acc[q][z] = 0.f;
    }
    const int clo = max(0, r0 - h), chi = min(L - 1, r0 + kSB - 1 + h);
    for (int t = clo / kSB; t <= chi / kSB; ++t) {
        const int c0 = t * kSB;
        __syncthreads();
        for (int e = threadIdx.x; e < kSB * d; e += kSNT) {
            int r = e / d, k = e - r * d;
            const size_t gi = size_t(c0 + r) * d + k;
            Ys[r * ld + k] = to_f(Y[gi]);
            if (has_dp) Bs[r * ld + k] = to_f(Bm[gi]);
            if (Z) Zs[r * ld + k] = to_f(Z[gi]);
        }
        if (threadIdx.x < kSB) {
            const int c = c0 + threadIdx.x;
            const bool act = logm[c] != neg_inf() && c != D;
            colv[threadIdx.x] = act ? p.pc[base + c] : neg_inf();
            colv[kSB + threadIdx.x] = p.m ? p.m[base + c] : 0.f;
            for (int k = 0; k < nm; ++k) colv[(2 + k) * kSB + threadIdx.x] = p.yc[k][base + c];
        }
        __syncthreads();
        const int c = c0 + lane;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int rl = warp * 4 + q, r = r0 + rl;
            float sacc = 0.f, dacc = 0.f;
            for (int k = 0; k < d; ++k) sacc = fmaf(Xs[rl * ld + k], Ys[lane * ld + k], sacc);
            if (has_dp)
                for (int k = 0; k < d; ++k) dacc = fmaf(As[rl * ld + k], Bs[lane * ld + k], dacc);
            float x = fmaf(sacc, sc, rowv[rl] + colv[lane]);
            const bool in = (abs(r - c) <= h) && logm[r] != neg_inf() && r != D && x != neg_inf();
            const float P = in ? expf(x) : 0.f;
            if (p.sout) {
                if (p.s_dp) s1[q] = fmaf(P, dacc, s1[q]);
                s2[q] = fmaf(P, colv[kSB + lane], s2[q]);
            }
            if (p.vout) {
                float mod = p.v_dp ? dacc : 1.f;
                for (int k = 0; k < nm; ++k) mod -= rowv[(3 + k) * kSB + rl] * colv[(2 + k) * kSB + lane];
                Cs[rl * 33 + lane] = P * mod;
            }
        }
        if (p.vout) {
            __syncthreads();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int rl = warp * 4 + q;
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                    const int zc = lane + 32 * z;
                    if (zc < d) {
                        float a = acc[q][z];
                        for (int cc = 0; cc < kSB; ++cc) a = fmaf(Cs[rl * 33 + cc], Zs[cc * ld + zc], a);
                        acc[q][z] = a;
                    }
                }
            }
        }
    }
    // Finish the rows: lane reductions, dustbin link, writes.
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int rl = warp * 4 + q, r = r0 + rl;
        if (p.sout) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                s1[q] += __shfl_xor_sync(0xffffffffu, s1[q], off);
                s2[q] += __shfl_xor_sync(0xffffffffu, s2[q], off);
            }
        }
        const bool ract = logm[r] != neg_inf();
        if (r == D && d_act) continue;   // dense dustbin row kernel
        float Pd = 0.f, dpd = 0.f, coefd = 0.f;
        if (ract && d_act) {
            Pd = expf(p.sd_term[base + r] + rowv[rl] + p.pc[base + D]);
            if (has_dp) dpd = p.dp_term[base + r];
            float mod = p.v_dp ? dpd : 1.f;
            for (int k = 0; k < nm; ++k) mod -= rowv[(3 + k) * kSB + rl] * p.yc[k][base + D];
            coefd = Pd * mod;
        }
        if (p.sout && lane == 0) {
            float a = s1[q], bb = s2[q];
            if (ract && d_act) {
                if (p.s_dp) a = fmaf(Pd, dpd, a);
                if (p.m) bb = fmaf(Pd, p.m[base + D], bb);
            }
            float outv = ract ? rowv[kSB + rl] * (a + rowv[2 * kSB + rl] * bb) : 0.f;
            if (!isfinite(outv)) atomicOr(p.status, kStatusNonFinite);
            p.sout[base + r] = outv;
        }
        if (p.vout) {
            T* vo = static_cast<T*>(p.vout) + (base + r) * d;
            const T* zD = d_act ? static_cast<const T*>(p.Z) + (base + D) * d : nullptr;
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const int zc = lane + 32 * z;
                if (zc < d) {
                    float a = acc[q][z];
                    if (ract && d_act) a = fmaf(coefd, to_f(zD[zc]), a);
                    vo[zc] = from_f<T>(ract ? p.vscale * a : 0.f);
                }
            }
        }
    }
}

// Dense dustbin row of a backward sweep (row r = D over every active real column, plus
// (D, D)).  CTA (split, unit) takes kDCols columns (column L stands for (D, D)); the last CTA
// of a unit to finish adds up the partial sums and vectors and writes the row's outputs.
template <typename T>
__global__ void __launch_bounds__(256) dustbin_bwd_kernel(BwdPass p) {
    const int split = blockIdx.x, ns = gridDim.x, bh = blockIdx.y, b = bh / p.g.H;
    const int L = p.g.L, D = p.g.D, d = p.g.d;
    const size_t base = size_t(bh) * L;
    const float* logm = p.logm + size_t(b) * L;
    if (D < 0 || logm[D] == neg_inf()) return;
    const int nm = p.nmod;
    const bool has_dp = (p.sout && p.s_dp) || (p.vout && p.v_dp);
    const float prD = p.pr[base + D];
    const int c_begin = split * kDCols, c_end = min(L + 1, c_begin + kDCols);
    __shared__ float cs[kDCols];
    __shared__ float red1[256], red2[256];
    __shared__ float vred[8][128];
    __shared__ int last;
    float a1 = 0.f, a2 = 0.f;
    for (int c = c_begin + threadIdx.x; c < c_begin + kDCols; c += blockDim.x) {
        float coef = 0.f;
        const bool self = (c == L) && p.g.dself;
        const bool band = (c < L) && c != D && logm[c] != neg_inf();
        if (c < c_end && (band || self)) {
            const int cc = self ? D : c;
            const float sv = self ? p.sd_term[base + D] : p.sd_dense[base + c];
            const float P = expf(sv + prD + p.pc[base + cc]);
            const float dp = has_dp ? (self ? p.dp_term[base + D] : p.dp_dense[base + c]) : 0.f;
            if (p.sout) {
                if (p.s_dp) a1 = fmaf(P, dp, a1);
                if (p.m) a2 = fmaf(P, p.m[base + cc], a2);
            }
            if (p.vout) {
                float mod = p.v_dp ? dp : 1.f;
                for (int k = 0; k < nm; ++k) mod -= p.xr[k][base + D] * p.yc[k][base + cc];
                coef = P * mod;
            }
        }
        cs[c - c_begin] = coef;
    }
    red1[threadIdx.x] = a1;
    red2[threadIdx.x] = a2;
    __syncthreads();
    for (int st = 128; st > 0; st >>= 1) {
        if (threadIdx.x < st) {
            red1[threadIdx.x] += red1[threadIdx.x + st];
            red2[threadIdx.x] += red2[threadIdx.x + st];
        }
        __syncthreads();
    }
    // vector part: warp w takes columns w, w + 8, ...; lane covers elements lane + 32 z of Z's row
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nz = (d + 31) / 32;
    if (p.vout) {
        const T* Z = static_cast<const T*>(p.Z) + base * d;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int j = warp; j < c_end - c_begin; j += 8) {
            const float cf = cs[j];
            if (cf == 0.f) continue;
            const int cj = c_begin + j;
            const T* zr = Z + size_t(cj == L ? D : cj) * d;
#pragma unroll
            for (int z = 0; z < 4; ++z)
                if (z < nz && lane + 32 * z < d) acc[z] = fmaf(cf, to_f(zr[lane + 32 * z]), acc[z]);
        }
#pragma unroll
        for (int z = 0; z < 4; ++z)
            if (z < nz && lane + 32 * z < d) vred[warp][lane + 32 * z] = acc[z];
    }
    __syncthreads();
    const int pw = d + 2;
    float* part = p.dpart + size_t(bh) * ns * pw + size_t(split) * pw;
    if (threadIdx.x == 0) {
        part[0] = red1[0];
        part[1] = red2[0];
    }
    if (p.vout && threadIdx.x < d) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += vred[w][threadIdx.x];
        part[2 + threadIdx.x] = v;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(p.dcnt + bh, 1u) == unsigned(ns - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    const float* parts = p.dpart + size_t(bh) * ns * pw;
    // The unit's partials, merged by the whole block in a fixed order (deterministic): the scalars
    // by a strided sum and a tree, the vector by G = blockDim.x / d groups of d threads, group g
    // summing partials g, g + G, ..., the groups then added in order.
    if (p.sout) {
        float s1 = 0.f, s2 = 0.f;
        for (int i = threadIdx.x; i < ns; i += blockDim.x) {
            s1 += __ldcg(parts + size_t(i) * pw);
            s2 += __ldcg(parts + size_t(i) * pw + 1);
        }
        red1[threadIdx.x] = s1;
        red2[threadIdx.x] = s2;
    }
    __syncthreads();
    if (p.sout) {
        for (int st = 128; st > 0; st >>= 1) {
            if (threadIdx.x < st) {
                red1[threadIdx.x] += red1[threadIdx.x + st];
                red2[threadIdx.x] += red2[threadIdx.x + st];
            }
            __syncthreads();
        }
        if (threadIdx.x == 0) {
            const float outv = (p.f ? p.f[base + D] : 1.f) * (red1[0] + (p.hv ? p.hv[base + D] : 0.f) * red2[0]);
            if (!isfinite(outv)) atomicOr(p.status, kStatusNonFinite);
            p.sout[base + D] = outv;
        }
    }
    if (p.vout) {
        const int G = int(blockDim.x) / d, g = int(threadIdx.x) / d, e = int(threadIdx.x) - g * d;
        float a = 0.f;
        if (g < G)
            for (int i = g; i < ns; i += G) a += __ldcg(parts + size_t(i) * pw + 2 + e);
        float* vsum = &vred[0][0];                     // (free again: the block's own part is written)
        __syncthreads();
        if (g < G) vsum[g * d + e] = a;
        __syncthreads();
        if (threadIdx.x < d) {
            float v = 0.f;
            for (int k = 0; k < G; ++k) v += vsum[k * d + threadIdx.x];
            static_cast<T*>(p.vout)[(base + D) * d + threadIdx.x] = from_f<T>(p.vscale * v);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) p.dcnt[bh] = 0u;   // ready for the next launch of this call
}

// ---------------------------------------------------------------------------------------
// Backward vector preparation (§2.2: orbit factors exp(u(k)-u(R)), exp(v(k)-v(R)))
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_vectors_kernel(BwdVecArgs a) {
    const int bh = blockIdx.y, b = bh / a.H;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.L) return;
    const size_t L = size_t(a.L);
    const size_t idx = size_t(bh) * L + i;
    const float lm = a.logm[size_t(b) * L + i];
    const bool act = lm != neg_inf();
    const int R = a.R;
    auto U = [&](int k) { return a.u_tail[(size_t(bh) * (R + 1) + k) * L + i]; };
    auto Vv = [&](int k) { return a.v_tail[(size_t(bh) * (R + 1) + k) * L + i]; };
    auto AL = [&](int k) { return a.alpha[size_t(k) * a.BH * L + idx]; };
    auto BE = [&](int k) { return a.beta[size_t(k) * a.BH * L + idx]; };
    float pr = 0.f, pc = 0.f, f = 1.f, hv = 0.f, m = 0.f;
    float xr[kMaxMods], yc[kMaxMods];
    int nm = 0;
    if (act) {
        const float ea = expf(lm), ia = expf(-lm);
        const float uR = U(R), vR = Vv(R);
        switch (a.kind) {
            case kPassOut: pr = uR - lm; pc = vR; break;
            case kPassC1: pr = vR; pc = uR - lm; break;
            case kPassR2: pr = uR - lm; pc = vR; hv = -ea; m = BE(R) * ia; break;
            case kPassCk:
                pr = vR; pc = uR; hv = 1.f;
                f = -expf(Vv(a.k) - vR);
                m = expf(U(a.k + 1) - uR) * AL(a.k + 1) * ia;
                break;
            case kPassRk:
                pr = uR; pc = vR; hv = 1.f;
                f = -expf(U(a.k) - uR);
                m = expf(Vv(a.k) - vR) * BE(a.k) * ia;
                break;
            case kPassRF:
                pr = uR - lm; pc = vR;
                for (int k = 1; k <= R; ++k) {
                    const float eu = expf(U(k) - uR);
                    xr[nm] = ea * eu;                 yc[nm++] = expf(Vv(k) - vR) * BE(k) * ia;
                    xr[nm] = eu * AL(k);              yc[nm++] = expf(Vv(k - 1) - vR);
                }
                break;
            case kPassCF:
                pr = vR; pc = uR - lm;
                for (int k = 1; k <= R; ++k) {
                    const float eu = expf(U(k) - uR);
                    xr[nm] = expf(Vv(k) - vR) * BE(k) * ia;   yc[nm++] = ea * eu;
                    xr[nm] = expf(Vv(k - 1) - vR);            yc[nm++] = eu * AL(k);
                }
                break;
        }
    } else {
        if (a.kind == kPassRF || a.kind == kPassCF) {
            for (int k = 0; k < 2 * R; ++k) { xr[k] = 0.f; yc[k] = 0.f; }
            nm = 2 * R;
        }
    }
    a.pr[idx] = pr;
    a.pc[idx] = pc;
    if (a.pcm2) a.pcm2[idx] = (act && i != a.D) ? pc * kLog2e : neg_inf();
    if (a.f) a.f[idx] = f;
    if (a.hv) a.hv[idx] = hv;
    if (a.m) a.m[idx] = m;
    if (a.cext && (a.kind == kPassR2 || a.kind == kPassCk || a.kind == kPassRk))
        band_ext_row(a.cext + idx * 16, (act && i != a.D) ? pc * kLog2e : neg_inf(), a.isl2);
    if (a.kind == kPassR2 && a.s1part && a.sadd) {
        float t = 0.f;
        if (act)
            for (int sl = 0; sl < a.s1slots; ++sl) t += a.s1part[size_t(sl) * a.s1stride + idx];
        a.sadd[idx] = t;
    }
    for (int k = 0; k < nm; ++k) {
        a.xr[size_t(k) * a.BH * L + idx] = xr[k];
        a.yc[size_t(k) * a.BH * L + idx] = yc[k];
    }
    if ((a.kind == kPassRF || a.kind == kPassCF) && a.xext && a.yext && nm <= kMaxFoldMods) {
        alignas(16) __nv_bfloat16 xe[16];
        alignas(16) __nv_bfloat16 ye[16];
        const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
#pragma unroll
        for (int j = 0; j < 16; ++j) xe[j] = ye[j] = z;
        for (int k = 0; k < nm; ++k) {
            const float x = -xr[k], y = yc[k];
            const __nv_bfloat16 xh = __float2bfloat16_rn(x), yh = __float2bfloat16_rn(y);
            const __nv_bfloat16 xl = __float2bfloat16_rn(x - __bfloat162float(xh));
            const __nv_bfloat16 yl = __float2bfloat16_rn(y - __bfloat162float(yh));
            xe[3 * k] = xh; xe[3 * k + 1] = xh; xe[3 * k + 2] = xl;
            ye[3 * k] = yh; ye[3 * k + 1] = yl; ye[3 * k + 2] = yh;
        }
        uint4* xo = reinterpret_cast<uint4*>(a.xext + idx * 16);
        uint4* yo = reinterpret_cast<uint4*>(a.yext + idx * 16);
        xo[0] = *reinterpret_cast<const uint4*>(xe);
        xo[1] = *reinterpret_cast<const uint4*>(xe + 8);
        yo[0] = *reinterpret_cast<const uint4*>(ye);
        yo[1] = *reinterpret_cast<const uint4*>(ye + 8);
    }
}

// ---------------------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------------------
cudaError_t launch_prep_marginals(const Geom& g, const uint8_t* mask, int dustbin, float mass, float* logm,
                                  uint32_t* status, cudaStream_t st, uint32_t* bits, float* bias2) {
    if (g.B == 0 || g.L == 0) return cudaSuccess;
    prep_marginals_kernel<<<dim3(g.B, (g.L + kPrepSlice - 1) / kPrepSlice), 1024, 0, st>>>(g, mask, dustbin, mass,
                                                                                          logm, status, bits, bias2);
    return cudaGetLastError();
}

cudaError_t launch_dustbin_dots(const Geom& g, const void* P, const void* Qm, float s1, float* term, float* dense,
                                cudaStream_t st) {
    dim3 grid((g.L + 31) / 32, g.BH);   // 32 rows (8 lanes each) per block
    if (g.dtype == EOT_BF16)
        prep_dustbin_dots_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            g, static_cast<const __nv_bfloat16*>(P), static_cast<const __nv_bfloat16*>(Qm), s1, term, dense);
    else
        prep_dustbin_dots_kernel<float><<<grid, 256, 0, st>>>(g, static_cast<const float*>(P),
                                                              static_cast<const float*>(Qm), s1, term, dense);
    return cudaGetLastError();
}

static size_t simt_lse_smem(int d) { return size_t(2 * kSB * (d + 1) + kSB) * sizeof(float); }
static size_t simt_bwd_smem(int d) {
    return size_t(5 * kSB * (d + 1) + kSB * 33 + (2 + kMaxMods) * kSB + (3 + kMaxMods) * kSB) * sizeof(float);
}

cudaError_t launch_simt_lse(const LsePass& p, cudaStream_t st) {
    dim3 grid(p.g.L / kSB, p.g.BH);
    const size_t smem = simt_lse_smem(p.g.d);
    cudaError_t e;
    if (p.g.dtype == EOT_BF16) {
        e = cudaFuncSetAttribute(simt_lse_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        simt_lse_kernel<__nv_bfloat16><<<grid, kSNT, smem, st>>>(p);
    } else {
        e = cudaFuncSetAttribute(simt_lse_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        simt_lse_kernel<float><<<grid, kSNT, smem, st>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess || p.g.D < 0) return e;
    return launch_dustbin_lse(p, st);
}

// ---------------------------------------------------------------------------------------
// Whole forward solve of one unit in one CTA (small problems on CUDA cores)
// ---------------------------------------------------------------------------------------
// The scores S_rc of the unit's band (|r - c| <= h) do not change between half-steps, so they
// are formed once, in fp32 with the same products as simt_lse_item, and kept in shared memory
// as sband[r * (2 h + 1) + (c - r + h)]; the log2 potential biases of both sides stay there too.
// Every half-step is then a band log-sum-exp over shared memory (groups of G threads per row
// or column, merged by shuffles), separated by __syncthreads() instead of a grid barrier.
constexpr int kResThreads = 1024;
constexpr int kResRB = 32;   // rows of Q per staging chunk while the scores are formed

size_t simt_resident_smem(int L, int h, int d) {
    const size_t stage = size_t(2 * kResRB + 2 * h) * size_t(d + 1);   // Q chunk + the K rows its band reaches
    return (size_t(L) * size_t(2 * h + 1) + 3 * size_t(L) + stage) * sizeof(float);
}

template <typename T>
__global__ void __launch_bounds__(kResThreads) simt_resident_kernel(LsePass g0, const void* Qp, const void* Kp,
                                                                     float* u_tail, float* v_tail, int Tb, int R) {
    extern __shared__ float sm[];
    const int L = g0.g.L, h = g0.g.h, d = g0.g.d, ld = 2 * h + 1;
    const int bh = blockIdx.x, b = bh / g0.g.H;
    float* sband = sm;
    float* lmb = sband + size_t(L) * ld;   // log marginals
    float* ub2 = lmb + L;                  // log2 e * u, -inf for inactive rows
    float* vb2 = ub2 + L;
    float* Qs = vb2 + L;                     // [kResRB][d + 1]
    float* Ks = Qs + kResRB * (d + 1);       // [kResRB + 2 h][d + 1]
    const size_t base = size_t(bh) * L, pb = size_t(bh) * g0.pstride;
    const T* Q = static_cast<const T*>(Qp) + base * d;
    const T* K = static_cast<const T*>(Kp) + base * d;
    for (int i = threadIdx.x; i < L; i += blockDim.x) {
        const float lm = g0.logm[size_t(b) * L + i];
        lmb[i] = lm;
        vb2[i] = lm != neg_inf() ? 0.f : neg_inf();   // v = 0
    }
    // scores of rows [r0, r0 + kResRB): Q rows and the K rows [r0 - h, r0 + kResRB + h) staged
    // in shared memory (row pitch d + 1: neighbouring columns fall in different banks)
    for (int r0 = 0; r0 < L; r0 += kResRB) {
        const int nr = min(kResRB, L - r0), k0 = r0 - h, nk = nr + 2 * h;
        __syncthreads();
        for (int e = threadIdx.x; e < nr * d; e += blockDim.x) {
            const int i = e / d, k = e - i * d;
            Qs[i * (d + 1) + k] = to_f(Q[size_t(r0 + i) * d + k]);
        }
        for (int e = threadIdx.x; e < nk * d; e += blockDim.x) {
            const int i = e / d, k = e - i * d, c = k0 + i;
            Ks[i * (d + 1) + k] = (c >= 0 && c < L) ? to_f(K[size_t(c) * d + k]) : 0.f;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < nr * ld; e += blockDim.x) {
            const int i = e / ld, j = e - i * ld;   // row r0 + i, column r0 + i - h + j = k0 + i + j
            const float* qa = Qs + i * (d + 1);
            const float* ka = Ks + (i + j) * (d + 1);
            float acc = 0.f;
            for (int k = 0; k < d; ++k) acc = fmaf(qa[k], ka[k], acc);
            sband[size_t(r0) * ld + e] = acc;
        }
    }
    __syncthreads();
    // G threads per row (a power of two dividing 32), groups strided over the rows
    int G = 1;
    while (G < 32 && G * 2 * L <= int(blockDim.x)) G *= 2;
    const int grp = threadIdx.x / G, gl = threadIdx.x % G, ngrp = blockDim.x / G;
    const float sl2 = g0.g.scale * kLog2e;
    // Small bands with one row per group: every thread keeps its band entries of row grp (row
    // half-steps) and of column grp (column half-steps) in registers for the whole solve, so a
    // half-step is one independent bias load per entry, the exponentials and a group reduction.
    constexpr int kResRegs = 12;
    const int ne = (ld + G - 1) / G;
    if (L <= ngrp && ne <= kResRegs) {
        const int rc = grp;                    // the row (and the column) of this group
        float srow[kResRegs], scol[kResRegs];
#pragma unroll
        for (int e = 0; e < kResRegs; ++e) {
            const int j = gl + e * G, c = rc - h + j;   // column of S_rc / row of S_cr
            const bool ok = e < ne && j < ld && rc < L && c >= 0 && c < L;
            srow[e] = ok ? sband[size_t(rc) * ld + j] * sl2 : 0.f;
            scol[e] = ok ? sband[size_t(c) * ld + (2 * h - j)] * sl2 : 0.f;
        }
        for (int hs = 0; hs < 2 * (Tb + R); ++hs) {
            const int it = hs >> 1;
            const int slot = it < Tb ? 0 : it - Tb + 1;
            const bool col = hs & 1;
            const float* bias = col ? ub2 : vb2;   // the other side's log2 potential
            float* outb = col ? vb2 : ub2;
            float* out = (col ? v_tail : u_tail) + pb + size_t(slot) * L;
            float x[kResRegs];
            float m = neg_inf();
#pragma unroll
            for (int e = 0; e < kResRegs; ++e) {
                const int j = gl + e * G, c = rc - h + j;
                const bool ok = e < ne && j < ld && rc < L && c >= 0 && c < L;
                x[e] = ok ? (col ? scol[e] : srow[e]) + bias[ok ? c : 0] : neg_inf();
                m = fmaxf(m, x[e]);
            }
            float s = 0.f;
            if (m != neg_inf()) {
#pragma unroll
                for (int e = 0; e < kResRegs; ++e) s += ptx::ex2(x[e] - m);   // ex2(-inf) = 0
            }
            for (int off = G / 2; off > 0; off >>= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, m, off), s2 = __shfl_xor_sync(0xffffffffu, s, off);
                lse2_merge(m, s, m2, s2);
            }
            if (rc < L && gl == 0) {
                const float lm = lmb[rc];
                float outv = 0.f, ob = neg_inf();
                if (lm != neg_inf()) {
                    outv = lm - (m + log2f(s)) * kLn2;
                    if (!isfinite(outv)) atomicOr(g0.status, kStatusNonFinite);
                    ob = outv * kLog2e;
                }
                outb[rc] = ob;
                out[rc] = outv;
            }
            __syncthreads();
        }
        return;
    }
    for (int hs = 0; hs < 2 * (Tb + R); ++hs) {
        const int it = hs >> 1;
        const int slot = it < Tb ? 0 : it - Tb + 1;
        const bool col = hs & 1;
        const float* bias = col ? ub2 : vb2;   // the other side's log2 potential
        float* outb = col ? vb2 : ub2;
        float* out = (col ? v_tail : u_tail) + pb + size_t(slot) * L;
        for (int r0 = 0; r0 < L; r0 += ngrp) {   // uniform trip count: the shuffles below see every lane
            const int r = r0 + grp;
            // this thread's band entries: the maximum first, then the shifted sum
            float m = neg_inf(), s = 0.f;
            auto term = [&](int j) {
                const int c = r - h + j;
                if (c < 0 || c >= L) return neg_inf();
                const float bc = bias[c];
                if (bc == neg_inf()) return neg_inf();
                // S_rc for a row half-step, S_cr (the same product) for a column half-step
                const float sv = col ? sband[size_t(c) * ld + (r - c + h)] : sband[size_t(r) * ld + j];
                return fmaf(sv, sl2, bc);
            };
            if (r < L) {
                for (int j = gl; j < ld; j += G) m = fmaxf(m, term(j));
                if (m != neg_inf())
                    for (int j = gl; j < ld; j += G) {
                        const float x = term(j);
                        if (x != neg_inf()) s += exp2f(x - m);
                    }
            }
            for (int off = G / 2; off > 0; off >>= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, m, off), s2 = __shfl_xor_sync(0xffffffffu, s, off);
                lse2_merge(m, s, m2, s2);
            }
            if (r < L && gl == 0) {
                const float lm = lmb[r];
                float outv = 0.f, ob = neg_inf();
                if (lm != neg_inf()) {
                    outv = lm - (m + log2f(s)) * kLn2;
                    if (!isfinite(outv)) atomicOr(g0.status, kStatusNonFinite);
                    ob = outv * kLog2e;
                }
                outb[r] = ob;
                out[r] = outv;
            }
        }
        __syncthreads();
    }
}

bool simt_resident_possible(const Geom& g) {
    if (g.D >= 0 || g.L <= 0 || g.d <= 0) return false;
    int dev = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return false;
    return simt_resident_smem(g.L, g.h, g.d) <= size_t(optin);
}

cudaError_t launch_simt_resident(const LsePass& row, const void* Q, const void* K, float* u_tail, float* v_tail, int T,
                                 int R, cudaStream_t st) {
    if (!simt_resident_possible(row.g)) return cudaErrorInvalidValue;
    const size_t smem = simt_resident_smem(row.g.L, row.g.h, row.g.d);
    auto launch = [&](auto kernel) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        kernel<<<row.g.BH, kResThreads, smem, st>>>(row, Q, K, u_tail, v_tail, T, R);
        return cudaGetLastError();
    };
    return row.g.dtype == EOT_BF16 ? launch(simt_resident_kernel<__nv_bfloat16>) : launch(simt_resident_kernel<float>);
}

cudaError_t launch_simt_lse_fused(const LsePass& row, const void* Q, const void* K, float* u_tail, float* v_tail,
                                  float* ub2, float* vb2, int T, int R, uint32_t* gbar, cudaStream_t st) {
    if (row.g.D >= 0 || !gbar) return cudaErrorInvalidValue;
    const size_t smem = simt_lse_smem(row.g.d);
    const int items = (row.g.L / kSB) * row.g.BH;
    int nhs = 2 * (T + R);
    auto launch = [&](auto kernel) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        int per_sm = 0, dev = 0, n_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kSNT, smem);
        if (e != cudaSuccess) return e;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        const int grid = std::max(1, std::min(items, per_sm * n_sm));
        LsePass r = row;
        void* args[] = {&r, const_cast<void**>(&Q), const_cast<void**>(&K), &u_tail, &v_tail, &ub2, &vb2, &nhs, &T, &gbar};
        return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3(grid), dim3(kSNT), args, smem, st);
    };
    return row.g.dtype == EOT_BF16 ? launch(simt_lse_fused_kernel<__nv_bfloat16>) : launch(simt_lse_fused_kernel<float>);
}

// The dense dustbin row of one part of a sequence (a sharded solve): per unit, the (max, sum)
// partial of x_c = S_Dc + colpot_c over the active real columns c in [lo, hi), natural-log units
// (sum_c exp(x_c - max)); (-inf, 0) when there is none.  (D, D) is left to the caller.
__global__ void __launch_bounds__(256) dustbin_part_kernel(LsePass p, int lo, int hi, float* part) {
    const int bh = blockIdx.x, b = bh / p.g.H, L = p.g.L, D = p.g.D;
    const size_t base = size_t(bh) * L;
    const size_t pb = size_t(bh) * p.pstride;
    const float* logm = p.logm + size_t(b) * L;
    float m = neg_inf(), s = 0.f;
    for (int c = lo + int(threadIdx.x); c < hi; c += blockDim.x) {
        if (c == D || logm[c] == neg_inf()) continue;
        lse2_add(m, s, (p.sd_dense[base + c] + p.colpot[pb + c]) * kLog2e);
    }
    __shared__ float sm_m[256], sm_s[256];
    sm_m[threadIdx.x] = m;
    sm_s[threadIdx.x] = s;
    __syncthreads();
    for (int st = 128; st > 0; st >>= 1) {
        if (threadIdx.x < st) {
            float a = sm_m[threadIdx.x], bb = sm_s[threadIdx.x];
            lse2_merge(a, bb, sm_m[threadIdx.x + st], sm_s[threadIdx.x + st]);
            sm_m[threadIdx.x] = a;
            sm_s[threadIdx.x] = bb;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        part[2 * bh] = sm_m[0] == neg_inf() ? neg_inf() : sm_m[0] * kLn2;
        part[2 * bh + 1] = sm_s[0];
    }
}

cudaError_t launch_dustbin_part(const LsePass& p, int lo, int hi, float* part, cudaStream_t st) {
    if (!p.sd_dense || !part || p.g.D < 0 || lo < 0 || hi < lo || hi > p.g.L) return cudaErrorInvalidValue;
    dustbin_part_kernel<<<p.g.BH, 256, 0, st>>>(p, lo, hi, part);
    return cudaGetLastError();
}

cudaError_t launch_dustbin_lse(const LsePass& p, cudaStream_t st) {
    if (!p.dpart || !p.dcnt) return cudaErrorInvalidValue;
    dustbin_lse_kernel<<<dim3(dustbin_splits(p.g.L), p.g.BH), 256, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_simt_bwd(const BwdPass& p, cudaStream_t st) {
    dim3 grid(p.g.L / kSB, p.g.BH);
    const size_t smem = simt_bwd_smem(p.g.d);
    cudaError_t e;
    if (p.g.dtype == EOT_BF16) {
        e = cudaFuncSetAttribute(simt_bwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        simt_bwd_kernel<__nv_bfloat16><<<grid, kSNT, smem, st>>>(p);
    } else {
        e = cudaFuncSetAttribute(simt_bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        simt_bwd_kernel<float><<<grid, kSNT, smem, st>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess || p.g.D < 0) return e;
    return launch_dustbin_bwd(p, st);
}

cudaError_t launch_dustbin_bwd(const BwdPass& p, cudaStream_t st) {
    if (!p.dpart || !p.dcnt || p.g.d > 128) return cudaErrorInvalidValue;
    const dim3 grid(dustbin_splits(p.g.L), p.g.BH);
    if (p.g.dtype == EOT_BF16)
        dustbin_bwd_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(p);
    else
        dustbin_bwd_kernel<float><<<grid, 256, 0, st>>>(p);
    return cudaGetLastError();
}

// Masked log2 bias of the zero potential: 0 for active non-dustbin positions, -inf else.
// log2(e) * pot (0 when pot is null), -inf for inactive positions and the dustbin.
__global__ void __launch_bounds__(256) init_bias2_kernel(Geom g, const float* logm, const float* pot, float* bias2) {
    const int bh = blockIdx.y, b = bh / g.H;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= g.L) return;
    const bool act = logm[size_t(b) * g.L + i] != neg_inf() && i != g.D;
    const size_t o = size_t(bh) * g.L + i;
    bias2[o] = act ? (pot ? pot[o] * kLog2e : 0.f) : neg_inf();
}

// Bit t of word w of batch row b: positions [128 t, 128 t + 128) hold an active token other
// than the dustbin (tiles without one contribute nothing to a band sum and are skipped).
// One 1024-thread block per word; warp k examines tile 32 w + k.
__global__ void __launch_bounds__(1024) tile_bits_kernel(Geom g, const float* logm, uint32_t* bits) {
    const int words = tile_words(g.L);
    const int b = blockIdx.x / words, w = blockIdx.x - b * words;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ uint32_t acc;
    if (threadIdx.x == 0) acc = 0u;
    __syncthreads();
    const int t = w * 32 + warp;
    bool any = false;
    if (t * 128 < g.L) {
        const float* lm = logm + size_t(b) * g.L + size_t(t) * 128;
        for (int i = lane; i < 128; i += 32) any |= lm[i] != neg_inf() && (t * 128 + i) != g.D;
    }
    const unsigned vote = __ballot_sync(0xffffffffu, any);
    if (lane == 0 && vote) atomicOr(&acc, 1u << warp);
    __syncthreads();
    if (threadIdx.x == 0) bits[blockIdx.x] = acc;
}

// Squared norms for the tail's bias certificate: out[0] += sum (a - b)^2, out[1] += sum a^2,
// accumulated in float64 (grid-stride loop, warp shuffles, one pair of atomics per block).
template <typename T>
__global__ void sq_norms_kernel(const T* __restrict__ a, const T* __restrict__ b, size_t n, double* out) {
    double sd = 0.0, sa = 0.0;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += size_t(gridDim.x) * blockDim.x) {
        const double x = to_f(a[i]), y = to_f(b[i]);
        sd = fma(x - y, x - y, sd);
        sa = fma(x, x, sa);
    }
    for (int o = 16; o > 0; o >>= 1) {
        sd += __shfl_down_sync(0xffffffffu, sd, o);
        sa += __shfl_down_sync(0xffffffffu, sa, o);
    }
    __shared__ double part[2][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    if (lane == 0) {
        part[0][warp] = sd;
        part[1][warp] = sa;
    }
    __syncthreads();
    if (warp == 0) {
        sd = lane < nw ? part[0][lane] : 0.0;
        sa = lane < nw ? part[1][lane] : 0.0;
        for (int o = 16; o > 0; o >>= 1) {
            sd += __shfl_down_sync(0xffffffffu, sd, o);
            sa += __shfl_down_sync(0xffffffffu, sa, o);
        }
        if (lane == 0) {
            atomicAdd(out, sd);
            atomicAdd(out + 1, sa);
        }
    }
}

cudaError_t launch_sq_norms(const void* a, const void* b, size_t n, int dtype, double* out, int n_sm,
                            cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(out, 0, 2 * sizeof(double), st);
    if (e != cudaSuccess || n == 0) return e;
    const int threads = 256;
    const size_t want = (n + threads - 1) / threads;
    const int blocks = int(std::min<size_t>(want, size_t(4) * size_t(n_sm)));
    if (dtype == EOT_BF16)
        sq_norms_kernel<<<blocks, threads, 0, st>>>(static_cast<const __nv_bfloat16*>(a),
                                                    static_cast<const __nv_bfloat16*>(b), n, out);
    else
        sq_norms_kernel<<<blocks, threads, 0, st>>>(static_cast<const float*>(a), static_cast<const float*>(b), n,
                                                    out);
    return cudaGetLastError();
}

// Projective contraction certificate of the band's strictly positive blocks (the summary's
// §2.4, second certificate: with Hilbert's projective metric the strictly positive active
// blocks of the Sinkhorn map contract).  For a positive block K = exp(S) the Birkhoff-Hopf
// ratio is tanh(Delta / 4), Delta = max over rows i, i' and columns j, j' of
// S_ij + S_i'j' - S_ij' - S_i'j = max over row pairs of the range over j of S_ij - S_i'j.
// One CTA per tile pair (I, J = I + o), |o| <= m (pairs wholly inside the band); the block is
// restricted to its active real tokens.  The 128 x 128 score block is formed in fp32 in shared
// memory (rows padded to 129 floats: the pair loop reads 32 different rows per warp).
constexpr int kCT = 128, kCThreads = 256, kCChunk = 32;

size_t contraction_smem() {
    return (size_t(kCT) * (kCT + 1) + 2 * size_t(kCT) * (kCChunk + 1)) * sizeof(float) + 2 * kCT * sizeof(int);
}

template <typename T>
__global__ void __launch_bounds__(kCThreads) contraction_kernel(ContractArgs a) {
    extern __shared__ float csm[];
    float* S = csm;                                  // [128][129]
    float* Qs = S + kCT * (kCT + 1);                 // [128][33]: one 32-column chunk of the row tile
    float* Ks = Qs + kCT * (kCChunk + 1);            // [128][33]: ... of the column tile
    int* ract = reinterpret_cast<int*>(Ks + kCT * (kCChunk + 1));
    int* cact = ract + kCT;
    __shared__ float wmax[kCThreads / 32];
    __shared__ int nact[2];
    const int I = blockIdx.x, oi = blockIdx.y, bh = blockIdx.z, b = bh / a.H;
    const int J = I + oi - a.m;
    const int tid = threadIdx.x;
    float* outp = a.kappa + (size_t(bh) * a.nT + I) * size_t(2 * a.m + 1) + oi;
    if (J < 0 || J >= a.nT) {
        if (tid == 0) *outp = -1.f;
        return;
    }
    const int r0 = I * kCT, c0 = J * kCT;
    if (tid < 2) nact[tid] = 0;
    __syncthreads();
    auto active = [&](int pos) -> int {
        if (pos >= a.L || (a.D >= 0 && pos >= a.D)) return 0;
        return a.mask == nullptr || a.mask[size_t(b) * a.L + pos] != 0;
    };
    {
        const int t = tid & (kCT - 1);
        const int f = active((tid < kCT ? r0 : c0) + t);
        (tid < kCT ? ract : cact)[t] = f;
        if (f) atomicAdd(&nact[tid < kCT ? 0 : 1], 1);
    }
    // S = scale Q_I K_J^T; thread (ty, tx) owns rows 8 ty .. 8 ty + 7 and columns tx + 16 j
    const T* Qg = static_cast<const T*>(a.Q) + size_t(bh) * a.L * a.d;
    const T* Kg = static_cast<const T*>(a.K) + size_t(bh) * a.L * a.d;
    const int ty = tid >> 4, tx = tid & 15;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    for (int k0 = 0; k0 < a.d; k0 += kCChunk) {
        __syncthreads();   // the previous chunk has been read
        for (int e = tid; e < kCT * kCChunk; e += kCThreads) {
            const int r = e / kCChunk, c = e % kCChunk, col = k0 + c;
            float qv = 0.f, kv = 0.f;
            if (col < a.d) {
                if (r0 + r < a.L) qv = to_f(Qg[size_t(r0 + r) * a.d + col]);
                if (c0 + r < a.L) kv = to_f(Kg[size_t(c0 + r) * a.d + col]);
            }
            Qs[r * (kCChunk + 1) + c] = qv;
            Ks[r * (kCChunk + 1) + c] = kv;
        }
        __syncthreads();
#pragma unroll 4
        for (int c = 0; c < kCChunk; ++c) {
            float qr[8], kc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) qr[i] = Qs[(8 * ty + i) * (kCChunk + 1) + c];
#pragma unroll
            for (int j = 0; j < 8; ++j) kc[j] = Ks[(tx + 16 * j) * (kCChunk + 1) + c];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(qr[i], kc[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) S[(8 * ty + i) * (kCT + 1) + tx + 16 * j] = a.scale * acc[i][j];
    __syncthreads();
    if (nact[0] == 0 || nact[1] == 0) {   // no block on this tile pair
        if (tid == 0) *outp = -1.f;
        return;
    }
    // Delta: warp w takes the partner rows i' = w, w + 8, ...; lane l the rows l + 32 s
    const int warp = tid >> 5, lane = tid & 31;
    float best = 0.f;
    for (int ip = warp; ip < kCT; ip += kCThreads / 32) {
        if (!ract[ip]) continue;
        for (int s = 0; s < kCT / 32; ++s) {
            const int i = lane + 32 * s;
            float mx = -INFINITY, mn = INFINITY;
            for (int j = 0; j < kCT; ++j) {
                if (!cact[j]) continue;
                const float dl = S[i * (kCT + 1) + j] - S[ip * (kCT + 1) + j];
                mx = fmaxf(mx, dl);
                mn = fminf(mn, dl);
            }
            if (ract[i]) best = fmaxf(best, mx - mn);
        }
    }
    for (int o = 16; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (lane == 0) wmax[warp] = best;
    __syncthreads();
    if (tid == 0) {
        float v = 0.f;
        for (int w = 0; w < kCThreads / 32; ++w) v = fmaxf(v, wmax[w]);
        *outp = tanhf(0.25f * v);
    }
}

cudaError_t launch_contraction(const ContractArgs& a, int dtype, int BH, cudaStream_t st) {
    if (a.m < 0 || a.nT == 0 || BH == 0) return cudaSuccess;
    const size_t smem = contraction_smem();
    const dim3 grid(a.nT, 2 * a.m + 1, BH);
    if (dtype == EOT_BF16) {
        cudaError_t e = cudaFuncSetAttribute(contraction_kernel<__nv_bfloat16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        contraction_kernel<__nv_bfloat16><<<grid, kCThreads, smem, st>>>(a);
    } else {
        cudaError_t e = cudaFuncSetAttribute(contraction_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem));
        if (e != cudaSuccess) return e;
        contraction_kernel<float><<<grid, kCThreads, smem, st>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_tile_bits(const Geom& g, const float* logm, uint32_t* bits, cudaStream_t st) {
    tile_bits_kernel<<<g.B * tile_words(g.L), 1024, 0, st>>>(g, logm, bits);
    return cudaGetLastError();
}

cudaError_t launch_init_bias2(const Geom& g, const float* logm, float* bias2, cudaStream_t st, const float* pot) {
    dim3 grid((g.L + 255) / 256, g.BH);
    init_bias2_kernel<<<grid, 256, 0, st>>>(g, logm, pot, bias2);
    return cudaGetLastError();
}

cudaError_t launch_bwd_vectors(const BwdVecArgs& a, cudaStream_t st) {
    dim3 grid((a.L + 255) / 256, a.BH);
    bwd_vectors_kernel<<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace eot
