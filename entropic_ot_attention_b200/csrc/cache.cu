// Staircase sweeps of the tail adjoint from a cached reference plan (measurement variant of the
// backward; the default recomputes the plan in every sweep).
//
// Method: "Blockwise Differentiable Sinkhorn Attention", technical summary (gist.science
// 2605.08123), §2.2: every staircase factor of the R-step adjoint is the one reference plan
// P = P(R,R) times per-row and per-column orbit factors, so the staircase vectors are banded
// matrix-vector products with P:
//     alpha_k = f_r * sum_c P_rc m_c           (row sweep,    m = e^{v(k) - v(R)} beta_k / a)
//     beta_k  = f_c * sum_r P_rc m_r           (column sweep, m = e^{u(k+1) - u(R)} alpha_{k+1} / a)
// The row sweep that forms alpha_R stores its plan entries Pt = P / a (row-scaled) as bf16 once,
// in a tile-relative band store: row r of row tile I keeps columns [128 I - h, 128 I + 127 + h] at
// pcache[r * cpitch + (c - 128 I + h)], cpitch = 2 h + 128 (h a multiple of 128, so every band tile
// lands inside the row's store; entries outside the band are stored as 0).  These kernels then
// stream it once per staircase sweep on CUDA cores instead of recomputing S and exp(S) on the
// tensor cores: the recompute-versus-cache choice is measured, not assumed.
#include "kernels.cuh"

namespace eot {

namespace {

__device__ __forceinline__ bool tbit(const uint32_t* bits, int t) { return (bits[t >> 5] >> (t & 31)) & 1u; }

// One warp per row: out_r = f_r hv_r a_r sum_c Pt_rc m_c over the band (a_r Pt = P).
__global__ void __launch_bounds__(256) cached_row_kernel(CachedSweep a) {
    const int warps = blockDim.x >> 5;
    const long gw = long(blockIdx.x) * warps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (gw >= long(a.BH) * a.L) return;
    const int bh = int(gw / a.L), r = int(gw - long(bh) * a.L), b = bh / a.H;
    const size_t base = size_t(bh) * a.L;
    const float lm = a.logm[size_t(b) * a.L + r];
    const uint32_t* bits = a.tile_bits + size_t(b) * tile_words(a.L);
    if (lm == neg_inf() || !tbit(bits, r >> 7)) {
        if (lane == 0) a.out[base + r] = 0.f;
        return;
    }
    const int r0 = r & ~127;
    const int c_lo = max(0, r - a.h), c_hi = min(a.L - 1, r + a.h);
    const __nv_bfloat16* prow = a.P + (base + r) * size_t(a.cpitch);
    const float* m = a.m + base;
    float acc = 0.f;
    // 8 entries (16 bytes) per lane per step over the row's whole store, masked to the band
    for (int o = lane * 8; o < a.cpitch; o += 256) {
        const int c = r0 - a.h + o;   // column of store entry o
        if (c + 7 < c_lo || c > c_hi) continue;
        if (!tbit(bits, max(c, 0) >> 7)) continue;   // tiles without an active token were never stored
        const uint4 u = *reinterpret_cast<const uint4*>(prow + o);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int cj = c + j;
            if (cj < c_lo || cj > c_hi) continue;
            const uint32_t bits16 = (w[j >> 1] >> ((j & 1) * 16)) & 0xffffu;
            acc = fmaf(__uint_as_float(bits16 << 16), m[cj], acc);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
        const float out = a.f[base + r] * a.hv[base + r] * expf(lm) * acc;
        if (!isfinite(out)) atomicOr(a.status, kStatusNonFinite);
        a.out[base + r] = out;
    }
}

// One warp per 64 columns (two per lane): out_c = f_c hv_c sum_r Pt_rc (a_r m_r) over the band.
__global__ void __launch_bounds__(256) cached_col_kernel(CachedSweep a) {
    const int warps = blockDim.x >> 5;
    const long gw = long(blockIdx.x) * warps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int groups = a.L / 64;
    if (gw >= long(a.BH) * groups) return;
    const int bh = int(gw / groups), cg = int(gw - long(bh) * groups), b = bh / a.H;
    const size_t base = size_t(bh) * a.L;
    const int c = cg * 64 + 2 * lane;   // this lane's columns c, c + 1
    const uint32_t* bits = a.tile_bits + size_t(b) * tile_words(a.L);
    float acc0 = 0.f, acc1 = 0.f;
    if (tbit(bits, c >> 7)) {
        const int r_lo = max(0, cg * 64 - a.h), r_hi = min(a.L - 1, cg * 64 + 63 + a.h);
        const float* m = a.m + base;
        const float* lmrow = a.logm + size_t(b) * a.L;
        for (int r = r_lo; r <= r_hi; ++r) {
            if (!tbit(bits, r >> 7)) {   // rows of a tile without an active token: never stored
                r = (r | 127);
                continue;
            }
            const int d0 = c - r, d1 = c + 1 - r;
            const bool in0 = d0 >= -a.h && d0 <= a.h, in1 = d1 >= -a.h && d1 <= a.h;
            if (!(in0 || in1)) continue;
            const float lm = lmrow[r];
            if (lm == neg_inf()) continue;
            const float wr = m[r] * expf(lm);
            const uint32_t pr = *reinterpret_cast<const uint32_t*>(a.P + (base + r) * size_t(a.cpitch) +
                                                                   (c - (r & ~127) + a.h));
            if (in0) acc0 = fmaf(__uint_as_float(pr << 16), wr, acc0);
            if (in1) acc1 = fmaf(__uint_as_float(pr & 0xffff0000u), wr, acc1);
        }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int cj = c + j;
        const float lm = a.logm[size_t(b) * a.L + cj];
        float out = 0.f;
        if (lm != neg_inf() && tbit(bits, cj >> 7)) {
            out = a.f[base + cj] * a.hv[base + cj] * (j ? acc1 : acc0);
            if (!isfinite(out)) atomicOr(a.status, kStatusNonFinite);
        }
        a.out[base + cj] = out;
    }
}

}  // namespace

bool cached_sweeps_supported(const Geom& g) {
    return g.dtype == EOT_BF16 && (g.d == 64 || g.d == 128) && g.D < 0 && g.h % 128 == 0;
}

cudaError_t launch_cached_sweep(const CachedSweep& a, bool column, cudaStream_t st) {
    if (!a.P || a.h % 128 != 0 || a.cpitch != 2 * a.h + 128) return cudaErrorInvalidValue;
    const int threads = 256, warps = threads / 32;
    if (column) {
        const long n = long(a.BH) * (a.L / 64);
        cached_col_kernel<<<unsigned((n + warps - 1) / warps), threads, 0, st>>>(a);
    } else {
        const long n = long(a.BH) * a.L;
        cached_row_kernel<<<unsigned((n + warps - 1) / warps), threads, 0, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace eot
