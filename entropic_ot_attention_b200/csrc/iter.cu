// Forward Sinkhorn iterations with one exponential per band entry per iteration (sm_100a).
//
// Method: "Blockwise Differentiable Sinkhorn Attention", technical summary (gist.science
// 2605.08123), §2.1: balanced log-domain Sinkhorn on the band,
//     u = log a - LSE_j (S + v),   v = log b - LSE_i (S + u).
// Iteration k starts from a row stabiliser p (any finite vector: the previous u) and v(k-1):
//     E_ij = exp(S_ij + p_i + v(k-1)_j)                 one exponential per band entry
//     r_i  = sum_j E_ij,          u(k) = p + log a - log r
//     c_j  = sum_i E_ij a_i / r_i = sum_i exp(S_ij + u(k)_i + v(k-1)_j)
//     v(k) = v(k-1) + log b - log c
// p cancels from u(k) exactly; it only keeps every E_ij at most about 1.  The column sums reuse
// E: E e^{u(k) - p} is the plan with u(k), the scaling-orbit identity of §2.2 used forward.
// The row sums are taken in registers; E is kept in shared memory as bf16 for the whole
// 128-row strip, and the column sums are the tensor-core product (a/r)^T E, with a/r split into
// a bf16 high and low part.
//
// A strip is 128 rows of one unit; its band columns are the 128-column tiles of the window
// [128 s - h, 128 s + 127 + h] that hold an active token.  SPLIT = 1: one CTA holds the strip's
// E.  SPLIT = 2 (wide bands): a cluster of two CTAs shares the strip; each takes one 64-column
// half of every window tile, two consecutive halves forming one 128-column "virtual tile" per
// MMA, and the two halves of every row sum meet through distributed shared memory.
//
// Column sums of a strip go to per-strip partials in global memory (no atomics: the summation
// order is fixed and results are deterministic).  After a grid-wide barrier every CTA finalises
// a slice of the columns (c_j = the partials of the strips whose window holds j, in strip
// order, then v), and a second grid-wide barrier orders the new v before the next iteration.
//
// Roles (608 threads): warp 0 TMA producer; warp 1 TMEM allocator and issuer of the score MMAs
// (S = Q K^T, Q copied into TMEM per strip by tcgen05.cp); warps 2..17 epilogue (warp w reads
// TMEM lane quadrant w % 4 and the 32 columns (w - 2) / 4 of each virtual tile); warp 18 issuer
// of the column-sum MMAs.  Every wait is bounded (ptx::mbar_wait).
#include <cudaTypedefs.h>

#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"

namespace eot {

namespace {

constexpr float kNegInfI = -__builtin_huge_valf();

template <int DH, int SPLIT>
struct IterCfg {
    // E capacity: SPLIT 1 holds NEV whole tiles; SPLIT 2 holds nine 64-column halves (the fifth
    // virtual slot's second half, never written, overlaps the ring: the column MMA reads it into
    // lanes whose results are not used).
    static constexpr int NEV = SPLIT == 1 ? (DH == 128 ? 3 : 5) : 5;
    static constexpr int NEH = SPLIT == 1 ? 2 * NEV : 9;
    static constexpr int MAXT = SPLIT == 1 ? NEV : 9;     // window tiles per strip
    static constexpr int NSK = SPLIT == 1 ? 3 : (DH == 128 ? 2 : 4);
    static constexpr int KATOMS = DH / 64;
    static constexpr int NV = 4;                            // column-vector slots
    static constexpr uint32_t EH = 128 * 64 * 2;           // half slot: 128 rows x 64 columns bf16
    static constexpr uint32_t ES = 2 * EH;                  // virtual slot
    static constexpr uint32_t RS = 128 * DH * 2;            // ring slot: 128 rows x DH bf16
    static constexpr uint32_t ATOM = 128 * 128;             // one 64-element atom column of 128 rows
    static constexpr uint32_t VB = 128 * 4;
    static constexpr uint32_t OFF_E = 0;
    static constexpr uint32_t OFF_RING = NEH * EH;
    static constexpr uint32_t OFF_W = OFF_RING + NSK * RS;          // column-MMA B operand: a / r
    static constexpr uint32_t WB = 2 * 16 * 128;                    // 2 K atoms x 16 rows x 128 B
    static constexpr uint32_t OFF_V = OFF_W + WB;
    static constexpr uint32_t OFF_RED = OFF_V + NV * VB;            // [2][4][128] row partials
    static constexpr uint32_t OFF_X = OFF_RED + 2 * 4 * 128 * 4;    // [2][128] the peer's row sums
    static constexpr uint32_t OFF_RV = OFF_X + 2 * 128 * 4;          // [2][previous u 128, log a 128]
    static constexpr uint32_t OFF_BITS = OFF_RV + 2 * 256 * 4;
    static constexpr int BITS_WORDS = 256;
    static constexpr uint32_t OFF_BAR = OFF_BITS + BITS_WORDS * 4;
    // rfull[NSK] rempty[NSK] vfull[NV] vempty[NV] sfull[2] sempty[2] qfree[2] wready dempty xfull[2] coldone[NEV]
    // redfull[2] redfree[2] rvfull[2] rvempty[2] wfree
    static constexpr uint32_t NBARS = 2 * NSK + 2 * NV + 2 + 2 + 2 + 2 + 2 + NEV + 9;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr size_t SMEM = 1024 + OFF_MISC + 64;
    // TMEM: two 128-column score buffers, two DH/2-column Q copies, NEV 16-column column sums
    static constexpr uint32_t TM_S = 0, TM_Q = 256, TM_D = 256 + DH;
    static constexpr uint32_t IDESC_S = ptx::idesc_bf16(128, 128, false, false);
    static constexpr uint32_t IDESC_C = ptx::idesc_bf16(128, 16, true, false);
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(TM_D + 16 * NEV <= 512, "tensor memory");
};

// Pairs of exponentials per 32-column chunk taken on the FMA pipe (ptx::exp2_fma_x2) instead of
// MUFU in blocks wholly inside the band.
#ifndef EOT_ITER_FMA_PAIRS
#define EOT_ITER_FMA_PAIRS 0
#endif
constexpr int kIterFmaPairs = EOT_ITER_FMA_PAIRS;
// Load the next virtual tile's scores from TMEM while the current one is exponentiated (costs a
// second 32-register score buffer per epilogue thread).
#ifndef EOT_ITER_PREFETCH
#define EOT_ITER_PREFETCH 0
#endif
constexpr bool kIterPrefetch = EOT_ITER_PREFETCH != 0;

// 20 warps: warpgroup 0 = TMA producer (warp 0), score-MMA issuer (warp 1), column-MMA issuer
// (warp 2), row warp (warp 3: merges the row sums, exchanges them with the peer CTA, forms u and
// a / r); warpgroups 1..4 = the 16 epilogue warps.  Launched at 96 registers a
// thread (640 x 96 = 61440); warpgroup 0 gives registers back (56 a thread) and the epilogue
// warpgroups take them (104 a thread): 128 x 56 + 512 x 104 = 60416 <= 61440, the launch's total
// (the host refuses the launch if the kernel was built with another register count).
constexpr int kIterThreads = 640;
constexpr int kIterLaunchRegs = 96;
constexpr int kIterColWarp = 2;
constexpr int kIterRowWarp = 3;
constexpr int kIterEpi0 = 4;          // first epilogue warp

struct IterArgs {
    int H, L, h, BH, nst, nw;   // nst = L / 128 strips per unit; nw = window tiles (partial stride)
    int n_items, ipc;           // items = BH * nst; items per CTA (SPLIT 1) or per cluster (SPLIT 2)
    int words;                  // tile-bit words per batch row
    float sl2;                  // scale * log2(e)
    const float* logm;          // [B, L]
    const uint32_t* tile_bits;  // [B][words]
    float* u_tail;
    float* v_tail;
    size_t pstride;             // (R + 1) L
    float* vb2;                 // [BH, L] masked log2 column bias, updated in place per iteration
    float* part;                // [BH][nst][nw][128] column partial sums
    uint32_t* gbar;             // two counters per iteration (strips done, finalise done)
    uint32_t* status;
    int k0, nk, T;              // iterations k0 .. k0 + nk - 1 (1-based), T base iterations
    int fused;                  // finalise inside, grid-wide barriers (cooperative launch)
};

// Potential slots of iteration k (1-based): the base overwrites slot 0, tail iteration m = k - T
// writes slot m and reads slot m - 1.
__host__ __device__ __forceinline__ int it_in_slot(int k, int T) { return k <= T + 1 ? 0 : k - T - 1; }
__host__ __device__ __forceinline__ int it_out_slot(int k, int T) { return k <= T ? 0 : k - T; }

__device__ __forceinline__ bool bit_of(const uint32_t* bits, int t) { return (bits[t >> 5] >> (t & 31)) & 1u; }

// Whether every tile of [lo, hi] (at most 32 tiles) holds an active token.
__device__ __forceinline__ bool all_bits(const uint32_t* bits, int lo, int hi) {
    const int w0 = lo >> 5, w1 = hi >> 5;
    if (w0 == w1) {
        const uint32_t m = (hi - lo == 31) ? 0xffffffffu : (((1u << (hi - lo + 1)) - 1u) << (lo & 31));
        return (bits[w0] & m) == m;
    }
    const uint32_t m0 = 0xffffffffu << (lo & 31), m1 = (hi & 31) == 31 ? 0xffffffffu : ((2u << (hi & 31)) - 1u);
    return (bits[w0] & m0) == m0 && (bits[w1] & m1) == m1;
}

// The active tiles of a strip's window (list index i -> tile), grouped into virtual tiles: tile
// vt(p, 0) (and vt(p, 1), the second half's tile for SPLIT 2; -1 when absent).  A window whose
// tiles are all active (the usual case) needs no list: tile i is t_lo + i.
template <int SPLIT>
struct StripTiles {
    int nv, n, t_lo;
    bool full;
    int list[9];
    __device__ void build(const uint32_t* bits, int lo, int hi) {
        t_lo = lo;
        full = all_bits(bits, lo, hi);
        if (full) {
            n = hi - lo + 1;
        } else {
            n = 0;
            for (int t = lo; t <= hi; ++t)
                if (bit_of(bits, t)) list[n++] = t;
        }
        nv = SPLIT == 1 ? n : (n + 1) / 2;
    }
    __device__ __forceinline__ int vt(int p, int h) const {
        const int i = SPLIT == 1 ? p : 2 * p + h;
        return i >= n ? -1 : (full ? t_lo + i : list[i]);
    }
};

struct Strip {
    int bh, b, s, t_lo, t_hi;
    size_t base;
};

__device__ __forceinline__ Strip decode_strip(const IterArgs& a, int item) {
    Strip st;
    st.bh = item / a.nst;
    st.s = item - st.bh * a.nst;
    st.b = st.bh / a.H;
    st.base = size_t(st.bh) * a.L;
    st.t_lo = max(0, 128 * st.s - a.h) / 128;
    st.t_hi = min(a.L - 1, 128 * st.s + 127 + a.h) / 128;
    return st;
}

// c_j and v(k) for the columns [c0, c1) of the flattened [BH, L] column index (§2.1 column step,
// from the partials of every strip whose window holds column j, in strip order).  Each thread
// takes two columns at a time so that all their partial loads are in flight together.
__device__ void finalize_columns(const IterArgs& a, int k, long c0, long c1, long tid, long nthreads) {
    const int vin = it_in_slot(k, a.T), vout = it_out_slot(k, a.T);
    const int reach_lo = (a.h + 127) / 128 + 1, reach_hi = a.h / 128 + 1;
    constexpr int kMaxReach = 11;   // reach_lo + reach_hi + 1 <= 11 for h <= 512 (windows of at most 9 tiles)
    constexpr int CU = 2;
    for (long i0 = c0 + tid; i0 < c1; i0 += CU * nthreads) {
        float pv[CU][kMaxReach];
        float vin_v[CU], lm_v[CU];
#pragma unroll
        for (int u = 0; u < CU; ++u) {
            const long idx = i0 + u * nthreads;
            lm_v[u] = kNegInfI;
            vin_v[u] = 0.f;
#pragma unroll
            for (int i = 0; i < kMaxReach; ++i) pv[u][i] = 0.f;
            if (idx >= c1) continue;
            const int bh = int(idx / a.L), j = int(idx - long(bh) * a.L), b = bh / a.H;
            lm_v[u] = a.logm[size_t(b) * a.L + j];
            if (lm_v[u] == kNegInfI) continue;
            vin_v[u] = a.v_tail[size_t(bh) * a.pstride + size_t(vin) * a.L + j];
            const uint32_t* bits = a.tile_bits + size_t(b) * a.words;
            const int t = j >> 7;
            const int s_lo = max(0, t - reach_lo), s_hi = min(a.nst - 1, t + reach_hi);
#pragma unroll
            for (int i = 0; i < kMaxReach; ++i) {
                const int s = s_lo + i;
                if (s <= s_hi && bit_of(bits, s)) {
                    const int tlo = max(0, 128 * s - a.h) / 128, thi = min(a.L - 1, 128 * s + 127 + a.h) / 128;
                    if (t >= tlo && t <= thi)
                        pv[u][i] = __ldcg(a.part + ((size_t(bh) * a.nst + s) * a.nw + (t - tlo)) * 128 + (j & 127));
                }
            }
        }
#pragma unroll
        for (int u = 0; u < CU; ++u) {
            const long idx = i0 + u * nthreads;
            if (idx >= c1 || lm_v[u] == kNegInfI) continue;
            float c = 0.f;
#pragma unroll
            for (int i = 0; i < kMaxReach; ++i) c += pv[u][i];
            const int bh = int(idx / a.L), j = int(idx - long(bh) * a.L);
            const float vnew = vin_v[u] + lm_v[u] - logf(c);
            if (!isfinite(vnew)) atomicOr(a.status, kStatusNonFinite);
            a.v_tail[size_t(bh) * a.pstride + size_t(vout) * a.L + j] = vnew;
            a.vb2[size_t(bh) * a.L + j] = vnew * kLog2e;
        }
    }
}

template <int DH, int SPLIT>
__global__ void __launch_bounds__(kIterThreads, 1)
    tc_iter_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const IterArgs a) {
    using C = IterCfg<DH, SPLIT>;
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = SPLIT == 2 ? int(ptx::cluster_rank()) : 0;
    const int cl = blockIdx.x / SPLIT;
    const int item0 = cl * a.ipc, item1 = min(a.n_items, item0 + a.ipc);
    const int L = a.L, h = a.h;

    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    const uint32_t bar0 = ptx::smem_u32(bars);
    auto rfull = [&](int i) { return bar0 + 8u * i; };
    auto rempty = [&](int i) { return bar0 + 8u * (C::NSK + i); };
    auto vfull = [&](int i) { return bar0 + 8u * (2 * C::NSK + i); };
    auto vempty = [&](int i) { return bar0 + 8u * (2 * C::NSK + C::NV + i); };
    auto sfull = [&](int i) { return bar0 + 8u * (2 * C::NSK + 2 * C::NV + i); };
    auto sempty = [&](int i) { return bar0 + 8u * (2 * C::NSK + 2 * C::NV + 2 + i); };
    auto qfree = [&](int i) { return bar0 + 8u * (2 * C::NSK + 2 * C::NV + 4 + i); };
    const uint32_t wready = bar0 + 8u * (2 * C::NSK + 2 * C::NV + 6);
    const uint32_t dempty = bar0 + 8u * (2 * C::NSK + 2 * C::NV + 7);
    auto xfull = [&](int i) { return bar0 + 8u * (2 * C::NSK + 2 * C::NV + 8 + i); };
    // coldone[p]: the column-sum MMAs of virtual tile p (E slot p) of a strip are done
    auto coldone = [&](int p) { return bar0 + 8u * (2 * C::NSK + 2 * C::NV + 10 + p); };
    const uint32_t bar1 = bar0 + 8u * (2 * C::NSK + 2 * C::NV + 10 + C::NEV);
    auto redfull = [&](int i) { return bar1 + 8u * i; };         // the 16 epilogue warps' row partials
    auto redfree = [&](int i) { return bar1 + 8u * (2 + i); };   // ... read by the row warp
    auto rvfull = [&](int i) { return bar1 + 8u * (4 + i); };    // row vectors of a strip landed
    auto rvempty = [&](int i) { return bar1 + 8u * (6 + i); };   // ... read by the epilogue and the row warp
    const uint32_t wfree = bar1 + 8u * 8;                        // a strip's column MMAs are done with W
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    // Tile bits of the batch rows this CTA's strips touch, in shared memory when they fit.
    uint32_t* sbits = reinterpret_cast<uint32_t*>(sm + C::OFF_BITS);
    const int b_first = item1 > item0 ? (item0 / a.nst) / a.H : 0;
    const int b_last = item1 > item0 ? ((item1 - 1) / a.nst) / a.H : -1;
    const int nbw = (b_last - b_first + 1) * a.words;
    const bool bits_in_smem = nbw <= C::BITS_WORDS;
    if (bits_in_smem)
        for (int i = tid; i < nbw; i += blockDim.x) sbits[i] = a.tile_bits[size_t(b_first) * a.words + i];
    const uint32_t* bits0 = bits_in_smem ? sbits : a.tile_bits + size_t(b_first) * a.words;
    auto bits_of = [&](int b) -> const uint32_t* { return bits0 + (b - b_first) * a.words; };
    // The column-MMA B operand holds a / r in rows 0 (high part) and 1 (low part); rows 2..15 stay 0.
    for (int i = tid; i < int(C::WB / 4); i += blockDim.x) reinterpret_cast<uint32_t*>(sm + C::OFF_W)[i] = 0u;

    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < C::NSK; ++i) { ptx::mbar_init(rfull(i), 1); ptx::mbar_init(rempty(i), 1); }
        for (int i = 0; i < C::NV; ++i) { ptx::mbar_init(vfull(i), 1); ptx::mbar_init(vempty(i), 16); }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(sfull(i), 1);
            ptx::mbar_init(sempty(i), 16);
            ptx::mbar_init(qfree(i), 1);
            ptx::mbar_init(xfull(i), 32);
            ptx::mbar_init(redfull(i), 16);
            ptx::mbar_init(redfree(i), 1);
            ptx::mbar_init(rvfull(i), 1);
            ptx::mbar_init(rvempty(i), 17);
        }
        ptx::mbar_init(wfree, 1);
        ptx::mbar_init(wready, 1);
        for (int p = 0; p < C::NEV; ++p) ptx::mbar_init(coldone(p), 1);
        ptx::mbar_init(dempty, 4);
        ptx::mbar_fence_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(misc), 512);
        ptx::tmem_relinquish();
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    if (SPLIT == 2) ptx::cluster_sync();   // the peer's barriers are initialised before any remote arrive
    ptx::tc_fence_after();
    const uint32_t tbase = misc[0];
    const int k_end = a.k0 + a.nk;

    if (warp < kIterEpi0) {
    // warpgroup 0 (control warps) gives registers back; every warp of it executes this
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;");
    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer: per strip Q, then this CTA's part of each virtual tile ----------------
            ptx::prefetch_tmap(&tmQ);
            ptx::prefetch_tmap(&tmK);
            int gr = 0, gv = 0, mr = 0;
            bool ok = true;
            for (int k = a.k0; k < k_end && ok; ++k) {
                // the column biases of iteration k are final once every CTA has finalised iteration k - 1
                bool vready = !a.fused || k == a.k0;
                for (int item = item0; item < item1 && ok; ++item) {
                    const Strip st = decode_strip(a, item);
                    const uint32_t* bits = bits_of(st.b);
                    if (!bit_of(bits, st.s)) continue;
                    StripTiles<SPLIT> tl;
                    tl.build(bits, st.t_lo, st.t_hi);
                    {
                        const int sl = gr % C::NSK;
                        if (!ptx::mbar_wait(rempty(sl), ((gr / C::NSK) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                        ptx::mbar_expect_tx(rfull(sl), C::RS);
                        const uint32_t dst = ptx::smem_u32(sm + C::OFF_RING + sl * C::RS);
                        for (int ka = 0; ka < C::KATOMS; ++ka)
                            ptx::tma_load_2d(dst + ka * C::ATOM, &tmQ, ka * 64, int(st.base) + 128 * st.s, rfull(sl));
                        ++gr;
                    }
                    if (!vready) {
                        const int j = k - a.k0;
                        if (!ptx::grid_wait(a.gbar + 2 * j - 1, gridDim.x, abort_flag, a.status)) { ok = false; break; }
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                        vready = true;
                    }
                    {
                        // the strip's row vectors: the previous u (the row stabiliser) and log a
                        const int rb = mr & 1;
                        if (!ptx::mbar_wait(rvempty(rb), ((mr >> 1) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                        ptx::mbar_expect_tx(rvfull(rb), 1024);
                        const uint32_t rvd = ptx::smem_u32(sm + C::OFF_RV + rb * 1024);
                        ptx::bulk_load(rvd, a.u_tail + size_t(st.bh) * a.pstride + size_t(it_in_slot(k, a.T)) * L + 128 * st.s,
                                       512, rvfull(rb));
                        ptx::bulk_load(rvd + 512, a.logm + size_t(st.b) * L + 128 * st.s, 512, rvfull(rb));
                        ++mr;
                    }
                    for (int p = 0; p < tl.nv && ok; ++p) {
                        const int sl = gr % C::NSK;
                        if (!ptx::mbar_wait(rempty(sl), ((gr / C::NSK) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                        const uint32_t dst = ptx::smem_u32(sm + C::OFF_RING + sl * C::RS);
                        if (SPLIT == 1) {
                            ptx::mbar_expect_tx(rfull(sl), C::RS);
                            for (int ka = 0; ka < C::KATOMS; ++ka)
                                ptx::tma_load_2d(dst + ka * C::ATOM, &tmK, ka * 64, int(st.base) + 128 * tl.vt(p, 0), rfull(sl));
                        } else {
                            const bool two = tl.vt(p, 1) >= 0;
                            ptx::mbar_expect_tx(rfull(sl), two ? C::RS : C::RS / 2);
                            for (int ka = 0; ka < C::KATOMS; ++ka) {
                                ptx::tma_load_2d(dst + ka * C::ATOM, &tmK, ka * 64, int(st.base) + 128 * tl.vt(p, 0) + 64 * rank,
                                                 rfull(sl));
                                if (two)
                                    ptx::tma_load_2d(dst + ka * C::ATOM + 64 * 128, &tmK, ka * 64,
                                                     int(st.base) + 128 * tl.vt(p, 1) + 64 * rank, rfull(sl));
                            }
                        }
                        ++gr;
                        const int vs = gv % C::NV;
                        if (!ptx::mbar_wait(vempty(vs), ((gv / C::NV) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                        const uint32_t vd = ptx::smem_u32(sm + C::OFF_V + vs * C::VB);
                        if (SPLIT == 1) {
                            ptx::mbar_expect_tx(vfull(vs), C::VB);
                            ptx::bulk_load(vd, a.vb2 + st.base + 128 * tl.vt(p, 0), C::VB, vfull(vs));
                        } else {
                            const bool two = tl.vt(p, 1) >= 0;
                            ptx::mbar_expect_tx(vfull(vs), two ? C::VB : C::VB / 2);
                            ptx::bulk_load(vd, a.vb2 + st.base + 128 * tl.vt(p, 0) + 64 * rank, C::VB / 2, vfull(vs));
                            if (two) ptx::bulk_load(vd + C::VB / 2, a.vb2 + st.base + 128 * tl.vt(p, 1) + 64 * rank, C::VB / 2, vfull(vs));
                        }
                        ++gv;
                    }
                }
            }
            if (*abort_flag) {
                // every copy already issued lands before the CTA retires
                volatile int dummy = 0;
                for (int i = max(0, gr - C::NSK); i < gr; ++i) ptx::mbar_wait(rfull(i % C::NSK), (i / C::NSK) & 1, &dummy, a.status);
                for (int i = max(0, gv - C::NV); i < gv; ++i) ptx::mbar_wait(vfull(i % C::NV), (i / C::NV) & 1, &dummy, a.status);
                for (int i = max(0, mr - 2); i < mr; ++i) ptx::mbar_wait(rvfull(i & 1), (i >> 1) & 1, &dummy, a.status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- score MMAs: Q (copied into TMEM) times this CTA's K columns ----------------
            int gr = 0, gs = 0, m = 0;
            bool ok = true;
            for (int k = a.k0; k < k_end && ok; ++k)
            for (int item = item0; item < item1 && ok; ++item) {
                const Strip st = decode_strip(a, item);
                const uint32_t* bits = bits_of(st.b);
                if (!bit_of(bits, st.s)) continue;
                StripTiles<SPLIT> tl;
                tl.build(bits, st.t_lo, st.t_hi);
                const int qb = m & 1;
                const uint32_t qtm = tbase + C::TM_Q + uint32_t(qb * (DH / 2));
                {
                    const int sl = gr % C::NSK;
                    if (!ptx::mbar_wait(rfull(sl), (gr / C::NSK) & 1, abort_flag, a.status)) { ok = false; break; }
                    // the strip two places back, which read this Q buffer, is done with it
                    if (m >= 2 && !ptx::mbar_wait(qfree(qb), ((m - 2) >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t src = ptx::smem_u32(sm + C::OFF_RING + sl * C::RS);
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk)
                        ptx::tmem_cp_128x256b(qtm + uint32_t(kk * 8),
                                              ptx::smem_desc(src + (kk >> 2) * C::ATOM + (kk & 3) * 32, 16, 1024));
                    ptx::mma_commit(rempty(sl));
                    ++gr;
                }
                for (int p = 0; p < tl.nv && ok; ++p) {
                    const int sl = gr % C::NSK, buf = gs & 1;
                    if (!ptx::mbar_wait(rfull(sl), (gr / C::NSK) & 1, abort_flag, a.status)) { ok = false; break; }
                    if (!ptx::mbar_wait(sempty(buf), ((gs >> 1) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint64_t bd = ptx::smem_desc(ptx::smem_u32(sm + C::OFF_RING + sl * C::RS), 16, 1024);
                    const uint32_t dt = tbase + C::TM_S + uint32_t(buf * 128);
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk) {
                        const uint64_t koff = uint64_t(((kk >> 2) * C::ATOM + (kk & 3) * 32) >> 4);
                        ptx::mma_bf16_ts(dt, qtm + uint32_t(kk * 8), bd + koff, C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(sfull(buf));
                    ptx::mma_commit(rempty(sl));
                    ++gr;
                    ++gs;
                }
                if (!ok) break;
                ptx::mma_commit(qfree(qb));
                ++m;
            }
            if (*abort_flag && gs > 0) {
                volatile int dummy = 0;
                ptx::mbar_wait(sfull((gs - 1) & 1), ((gs - 1) >> 1) & 1, &dummy, a.status);
            }
        }
    } else if (warp == kIterColWarp) {
        if (lane == 0) {
            // ---------------- column sums: D_p = E_p^T (a / r) per virtual tile ----------------
            int m = 0, last_nv = 0;
            int cnt[C::NEV];
#pragma unroll
            for (int p = 0; p < C::NEV; ++p) cnt[p] = 0;
            bool ok = true;
            for (int k = a.k0; k < k_end && ok; ++k)
            for (int item = item0; item < item1 && ok; ++item) {
                const Strip st = decode_strip(a, item);
                const uint32_t* bits = bits_of(st.b);
                if (!bit_of(bits, st.s)) continue;
                StripTiles<SPLIT> tl;
                tl.build(bits, st.t_lo, st.t_hi);
                if (!ptx::mbar_wait(wready, m & 1, abort_flag, a.status)) { ok = false; break; }
                if (m >= 1 && !ptx::mbar_wait(dempty, (m - 1) & 1, abort_flag, a.status)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t es = ptx::smem_u32(sm + C::OFF_E), ws = ptx::smem_u32(sm + C::OFF_W);
                for (int p = 0; p < tl.nv; ++p) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        // A = E^T: M = the virtual tile's 128 columns (two 64-column atoms EH apart),
                        // K = the strip's 128 rows, 16 per step (2048 bytes); B = a / r, K-major.
                        const uint64_t ad = ptx::smem_desc(es + uint32_t(p) * C::ES + uint32_t(kk) * 2048u, C::EH, 1024);
                        const uint64_t bd = ptx::smem_desc(ws + uint32_t(kk >> 2) * 2048u + uint32_t(kk & 3) * 32u, 16, 1024);
                        ptx::mma_bf16(tbase + C::TM_D + uint32_t(16 * p), ad, bd, C::IDESC_C, kk > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(coldone(p));   // E slot p is free, D_p is ready
                }
                ptx::mma_commit(wfree);   // the strip's column MMAs no longer read W
#pragma unroll
                for (int p = 0; p < C::NEV; ++p) cnt[p] += p < tl.nv ? 1 : 0;
                last_nv = tl.nv;
                ++m;
            }
            if (*abort_flag && last_nv > 0) {
                // the last commit covers every MMA this thread issued
                volatile int dummy = 0;
                int c = 0;
#pragma unroll
                for (int p = 0; p < C::NEV; ++p) c = p == last_nv - 1 ? cnt[p] : c;
                ptx::mbar_wait(coldone(last_nv - 1), (c - 1) & 1, &dummy, a.status);
            }
        }
    } else if (warp == kIterRowWarp) {
        // ---------------- row warp: per strip, r = the four column groups' row sums (plus the peer
        // CTA's half for SPLIT 2, added in rank order), u = p + log a - log r, and a / r for the
        // column-sum MMAs; rows lane + 32 i, i = 0..3 ----------------
        const float* red = reinterpret_cast<const float*>(sm + C::OFF_RED);
        float* xbuf = reinterpret_cast<float*>(sm + C::OFF_X);
        const float* rv = reinterpret_cast<const float*>(sm + C::OFF_RV);
        const uint32_t peer = uint32_t(rank ^ 1);
        int m = 0;
        bool ok = true;
        for (int k = a.k0; k < k_end; ++k) {
            const int so = it_out_slot(k, a.T);
            for (int item = item0; item < item1; ++item) {
                const Strip st = decode_strip(a, item);
                if (!bit_of(bits_of(st.b), st.s)) continue;
                const int rb = m & 1;
                bool w = ok && ptx::mbar_wait(redfull(rb), (m >> 1) & 1, abort_flag, a.status);
                w = w && ptx::mbar_wait(rvfull(rb), (m >> 1) & 1, abort_flag, a.status);
                // the previous strip's column MMAs no longer read W
                w = w && (m == 0 || ptx::mbar_wait(wfree, (m - 1) & 1, abort_flag, a.status));
                if (!__all_sync(0xffffffffu, w)) ok = false;
                float rs[4];
                const float* rd = red + rb * 512;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int rr = lane + 32 * i;
                    rs[i] = (rd[rr] + rd[128 + rr]) + (rd[256 + rr] + rd[384 + rr]);
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(redfree(rb));
                if (SPLIT == 2) {
                    // exchange the halves of the row sums with the peer CTA
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        ptx::st_cluster_f32(ptx::mapa(ptx::smem_u32(xbuf + rb * 128 + lane + 32 * i), peer), rs[i]);
                    ptx::mbar_arrive_cluster(ptx::mapa(xfull(rb), peer));
                    const bool w4 = ok && ptx::mbar_wait_cluster(xfull(rb), (m >> 1) & 1, abort_flag, a.status);
                    if (!__all_sync(0xffffffffu, w4)) ok = false;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float other = xbuf[rb * 128 + lane + 32 * i];
                        rs[i] = rank == 0 ? rs[i] + other : other + rs[i];
                    }
                }
                const size_t pb = size_t(st.bh) * a.pstride;
                for (int i = 0; i < 4; ++i) {
                    const int rr = lane + 32 * i;
                    const float uold = rv[rb * 256 + rr], lm = rv[rb * 256 + 128 + rr];
                    float unew = 0.f, wv = 0.f;
                    if (lm != kNegInfI) {
                        unew = uold + lm - logf(rs[i]);
                        if (!isfinite(unew)) atomicOr(a.status, kStatusNonFinite);
                        wv = rs[i] > 0.f ? expf(lm) / rs[i] : 0.f;
                    }
                    if (rank == 0 && ok) a.u_tail[pb + size_t(so) * L + 128 * st.s + rr] = unew;
                    // a / r as a bf16 high / low pair: rows n = 0, 1 of the K-major B operand
                    const __nv_bfloat16 whi = __float2bfloat16_rn(wv);
                    const __nv_bfloat16 wlo = __float2bfloat16_rn(wv - __bfloat162float(whi));
                    const int ii = rr & 63;
                    uint8_t* wb = sm + C::OFF_W + (rr >> 6) * 2048;
                    *reinterpret_cast<__nv_bfloat16*>(wb + 0 * 128 + (((ii >> 3) ^ 0) << 4) + (ii & 7) * 2) = whi;
                    *reinterpret_cast<__nv_bfloat16*>(wb + 1 * 128 + (((ii >> 3) ^ 1) << 4) + (ii & 7) * 2) = wlo;
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(rvempty(rb));
                    ptx::mbar_arrive(wready);
                }
                ++m;
            }
            // this CTA's u of iteration k precede its arrival on the grid-wide barrier
            if (a.fused) ptx::named_bar_sync(10, 512 + 32);
        }
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 104;");
        // ---------------- epilogue: 16 warps ----------------
        const int q = warp & 3;                 // TMEM lane quadrant (fixed by the warp's rank)
        const int g = (warp - kIterEpi0) >> 2;  // which 32 columns of every virtual tile
        const int row = q * 32 + lane;
        const uint32_t lane_base = uint32_t(q * 32) << 16;
        const uint32_t crow = uint32_t(row >> 3) * 1024u + uint32_t(row & 7) * 128u;
        const int etid = tid - 32 * kIterEpi0;  // 0 .. 511
        const uint64_t SL2 = ptx::f2(a.sl2, a.sl2);
        float* red = reinterpret_cast<float*>(sm + C::OFF_RED);
        const float* rv = reinterpret_cast<const float*>(sm + C::OFF_RV);
        const int half = SPLIT == 2 ? (g >> 1) : 0;
        int m = 0, gs = 0, gv = 0;
        // completions of coldone[p] expected so far (one per strip that used E slot p)
        int cnt[C::NEV];
#pragma unroll
        for (int p = 0; p < C::NEV; ++p) cnt[p] = 0;
        auto slot_count = [&](int p) {
            int c = 0;
#pragma unroll
            for (int i = 0; i < C::NEV; ++i) c = i == p ? cnt[i] : c;
            return c;
        };
        bool ok = true;
        // the previous strip, whose column sums are read out at the end of the next strip (warps g == 3)
        bool have_prev = false;
        Strip prev{};
        StripTiles<SPLIT> prev_tl;
        prev_tl.nv = 0;
        prev_tl.n = 0;
        auto readout = [&]() {
            // D rows are the virtual tile's columns: lane 32 q + l of D_p.  All loads are issued
            // before one wait.
            const int mrow = q * 32 + lane;
            bool w = ok;
            for (int p = 0; p < prev_tl.nv && w; ++p)
                w = ptx::mbar_wait(coldone(p), (slot_count(p) - 1) & 1, abort_flag, a.status);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                return;
            }
            ptx::tc_fence_after();
            float d[C::NEV][2];
#pragma unroll
            for (int p = 0; p < C::NEV; ++p)
                if (p < prev_tl.nv) ptx::tmem_ld32x2_nowait(tbase + lane_base + C::TM_D + uint32_t(16 * p), d[p][0], d[p][1]);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int p = 0; p < C::NEV; ++p) {
                if (p >= prev_tl.nv) continue;
                int t, col;
                if (SPLIT == 1) {
                    t = prev_tl.vt(p, 0);
                    col = mrow;
                } else {
                    t = prev_tl.vt(p, mrow < 64 ? 0 : 1);
                    col = 64 * rank + (mrow & 63);
                }
                if (t >= 0)
                    a.part[((size_t(prev.bh) * a.nst + prev.s) * a.nw + (t - prev.t_lo)) * 128 + col] = d[p][0] + d[p][1];
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(dempty);
        };
        for (int k = a.k0; k < k_end; ++k) {
            const int j = k - a.k0;
            if (a.fused && j > 0) {
                // every CTA has finalised iteration k - 1 (v, and u of the peer's strips)
                if (etid == 0 && ok && !ptx::grid_wait(a.gbar + 2 * j - 1, gridDim.x, abort_flag, a.status)) ok = false;
                ptx::named_bar_sync(9, 512);
                ok = ok && !*abort_flag;
            }
            for (int item = item0; item < item1; ++item) {
                const Strip st = decode_strip(a, item);
                const uint32_t* bits = bits_of(st.b);
                if (!bit_of(bits, st.s)) continue;
                StripTiles<SPLIT> tl;
                tl.build(bits, st.t_lo, st.t_hi);
                const int r = 128 * st.s + row;
                const int rb = m & 1;
                // the row stabiliser (previous u) and log a of this strip's rows
                float lm = kNegInfI, uold = 0.f;
                {
                    const bool w0 = ok && ptx::mbar_wait(rvfull(rb), (m >> 1) & 1, abort_flag, a.status);
                    if (!__all_sync(0xffffffffu, w0)) ok = false;
                    if (ok) {
                        uold = rv[rb * 256 + row];
                        lm = rv[rb * 256 + 128 + row];
                    }
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(rvempty(rb));
                }
                const bool ract = lm != kNegInfI;
                const float bu = ract ? uold * kLog2e : kNegInfI;
                const uint64_t BU2 = ptx::f2(bu, bu);
                uint64_t acc2 = ptx::f2(0.f, 0.f);
                const int rw = 128 * st.s + q * 32;
                auto classify = [&](int p, int& cc) {
                    const int tcol = tl.vt(p, half);
                    if (tcol < 0) return -1;   // absent half
                    cc = SPLIT == 1 ? 128 * tcol + 32 * g : 128 * tcol + 64 * rank + 32 * (g & 1);
                    const int dmin = cc - (rw + 31), dmax = cc + 31 - rw;
                    return (dmin > h || dmax < -h) ? 0 : ((dmax <= h && dmin >= -h) ? 1 : 2);
                };
                // One virtual tile: its scores arrive in `cur` (loaded by the previous step, or here
                // for the first tile); the next tile's scores are loaded into `nxt` while this one
                // is exponentiated.
                auto tile = [&](int p, float (&cur)[32], float (&nxt)[32]) {
                    const int vs = gv % C::NV, buf = gs & 1;
                    int cc = 0;
                    const int cls = classify(p, cc);
                    if (p == 0 || !kIterPrefetch) {
                        const bool w2 = ok && ptx::mbar_wait(sfull(buf), (gs >> 1) & 1, abort_flag, a.status);
                        if (!__all_sync(0xffffffffu, w2)) ok = false;
                        ptx::tc_fence_after();
                        if (ok && cls > 0) ptx::tmem_ld32(tbase + lane_base + C::TM_S + uint32_t(buf * 128 + 32 * g), cur);
                    }
                    ptx::tmem_wait_ld(cur);
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(sempty(buf));
                    if (kIterPrefetch && p + 1 < tl.nv) {
                        const int bufn = (gs + 1) & 1;
                        int ccn = 0;
                        const int clsn = classify(p + 1, ccn);
                        const bool wn = ok && ptx::mbar_wait(sfull(bufn), ((gs + 1) >> 1) & 1, abort_flag, a.status);
                        if (!__all_sync(0xffffffffu, wn)) ok = false;
                        ptx::tc_fence_after();
                        if (ok && clsn > 0) ptx::tmem_ld32(tbase + lane_base + C::TM_S + uint32_t(bufn * 128 + 32 * g), nxt);
                    }
                    const bool w1 = ok && ptx::mbar_wait(vfull(vs), (gv / C::NV) & 1, abort_flag, a.status);
                    if (!__all_sync(0xffffffffu, w1)) ok = false;
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                    if (ok && cls > 0) {
                        const uint32_t vaddr = ptx::smem_u32(sm + C::OFF_V + vs * C::VB) + uint32_t(32 * g * 4);
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 bv = ptx::ld_shared_f4(vaddr + 16u * j4);
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                const int kx = 2 * j4 + hh;
                                uint64_t xx = ptx::ffma2(ptx::f2(cur[2 * kx], cur[2 * kx + 1]), SL2,
                                                         hh ? ptx::f2(bv.z, bv.w) : ptx::f2(bv.x, bv.y));
                                xx = ptx::fadd2(xx, BU2);
                                float x0, x1;
                                ptx::f2split(xx, x0, x1);
                                if (cls == 2) {
                                    const int dl = cc + 2 * kx - r;   // column - row of entry 2 kx
                                    if (dl < -h || dl > h) x0 = kNegInfI;
                                    if (dl + 1 < -h || dl + 1 > h) x1 = kNegInfI;
                                }
                                float e0, e1;
                                if (kx < kIterFmaPairs && cls == 1) {
                                    ptx::exp2_fma_x2(x0, x1, e0, e1);
                                } else {
                                    e0 = ptx::ex2(x0);
                                    e1 = ptx::ex2(x1);
                                }
                                acc2 = ptx::fadd2(acc2, ptx::f2(e0, e1));
                                pk[kx] = ptx::pack_bf16(e0, e1);
                            }
                        }
                    }
                    // E slot p is free once the column MMAs of the last strip that used it are done.
                    {
                        const int c = slot_count(p);
                        if (c > 0) {
                            const bool w3 = ok && ptx::mbar_wait(coldone(p), (c - 1) & 1, abort_flag, a.status);
                            if (!__all_sync(0xffffffffu, w3)) ok = false;
                        }
                    }
                    if (ok && cls >= 0) {
                        // 128-byte-swizzled tile, row = strip row, 16-byte unit u at (u ^ (row & 7))
                        const uint32_t ebase = ptx::smem_u32(sm + C::OFF_E) + uint32_t(p) * C::ES + uint32_t(g >> 1) * C::EH + crow;
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const uint32_t unit = uint32_t((g & 1) * 4 + t);
                            ptx::st_shared_v4(ebase + ((unit ^ uint32_t(row & 7)) << 4), pk[4 * t], pk[4 * t + 1],
                                              pk[4 * t + 2], pk[4 * t + 3]);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(vempty(vs));
                    ++gs;
                    ++gv;
                };
                float va[32];
                if (kIterPrefetch) {
                    float vb[32];
                    for (int p = 0; p < tl.nv; p += 2) {
                        tile(p, va, vb);
                        if (p + 1 < tl.nv) tile(p + 1, vb, va);
                    }
                } else {
                    for (int p = 0; p < tl.nv; ++p) tile(p, va, va);
                }
                // E (generic-proxy writes) must be visible to the column MMAs; the row partials go
                // to the row warp
                ptx::fence_proxy_async_smem();
                float a0, a1;
                ptx::f2split(acc2, a0, a1);
                if (m >= 2) {
                    const bool w5 = ok && ptx::mbar_wait(redfree(rb), ((m >> 1) - 1) & 1, abort_flag, a.status);
                    if (!__all_sync(0xffffffffu, w5)) ok = false;
                }
                red[rb * 512 + g * 128 + row] = a0 + a1;
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(redfull(rb));
                // the previous strip's column sums (its column MMAs finished long ago)
                if (g == 3 && have_prev) {
                    if (ok) readout();
                    have_prev = false;
                }
#pragma unroll
                for (int p = 0; p < C::NEV; ++p) cnt[p] += p < tl.nv ? 1 : 0;
                if (g == 3) {
                    have_prev = true;
                    prev = st;
                    prev_tl = tl;
                }
                ++m;
            }
            // the last strip's column sums, before this CTA counts itself done with iteration k
            if (g == 3 && have_prev) {
                if (ok) readout();
                have_prev = false;
            }
            if (a.fused) {
                ptx::named_bar_sync(10, 512 + 32);   // with the row warp: its u writes are done
                if (etid == 0) {
                    __threadfence();
                    atomicAdd(a.gbar + 2 * j, 1u);
                    if (ok && !ptx::grid_wait(a.gbar + 2 * j, gridDim.x, abort_flag, a.status)) ok = false;
                }
                ptx::named_bar_sync(9, 512);
                ok = ok && !*abort_flag;
                if (ok) {
                    const long total = long(a.BH) * L, per = (total + gridDim.x - 1) / gridDim.x;
                    const long c0 = long(blockIdx.x) * per, c1 = min(total, c0 + per);
                    finalize_columns(a, k, c0, c1, etid, 512);
                }
                ptx::named_bar_sync(9, 512);
                if (etid == 0) {
                    __threadfence();
                    atomicAdd(a.gbar + 2 * j + 1, 1u);
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (SPLIT == 2) ptx::cluster_sync();   // no CTA leaves while its peer may still write to it
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tbase, 512);
    }
}

__global__ void __launch_bounds__(256) finalize_kernel(const IterArgs a, int k) {
    const long total = long(a.BH) * a.L;
    finalize_columns(a, k, 0, total, long(blockIdx.x) * blockDim.x + threadIdx.x, long(gridDim.x) * blockDim.x);
}

template <int DH, int SPLIT>
cudaError_t launch_iter_variant(const CUtensorMap& tmQ, const CUtensorMap& tmK, IterArgs a, cudaStream_t st) {
    using C = IterCfg<DH, SPLIT>;
    auto kernel = tc_iter_kernel<DH, SPLIT>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::SMEM));
    if (e != cudaSuccess) return e;
    // the register split inside the kernel assumes this launch allocation
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kIterLaunchRegs) return cudaErrorNotSupported;
    // grid: one CTA (or CTA pair) per SM (pair), as many as can be resident at once
    int units = sm_count();
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[2];
    int na = 0;
    cfg.blockDim = dim3(kIterThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    if (SPLIT == 2) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 2;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
        cfg.gridDim = dim3(2 * units);
        cfg.attrs = attr;
        cfg.numAttrs = na;
        int ncl = 0;
        e = cudaOccupancyMaxActiveClusters(&ncl, reinterpret_cast<const void*>(kernel), &cfg);
        if (e != cudaSuccess) return e;
        if (ncl < 1) return cudaErrorNotSupported;
        units = ncl;
    }
    units = std::max(1, std::min(units, a.n_items));
    a.ipc = (a.n_items + units - 1) / units;
    units = (a.n_items + a.ipc - 1) / a.ipc;
    cfg.gridDim = dim3(SPLIT * units);
    if (a.fused) {
        attr[na].id = cudaLaunchAttributeCooperative;
        attr[na].val.cooperative = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, tmQ, tmK, a);
}

template <int DH>
cudaError_t launch_iter_dh(int split, const CUtensorMap& tmQ, const CUtensorMap& tmK, const IterArgs& a, cudaStream_t st) {
    return split == 1 ? launch_iter_variant<DH, 1>(tmQ, tmK, a, st) : launch_iter_variant<DH, 2>(tmQ, tmK, a, st);
}

}  // namespace

int iter_split(const Geom& g) {
    if (g.dtype != EOT_BF16 || (g.d != 64 && g.d != 128) || g.D >= 0) return 0;
    const int nw = iter_window_tiles(g.L, g.h);
    const int max1 = g.d == 128 ? IterCfg<128, 1>::MAXT : IterCfg<64, 1>::MAXT;
    if (nw <= max1) return 1;
    if (nw <= (g.d == 128 ? IterCfg<128, 2>::MAXT : IterCfg<64, 2>::MAXT)) return 2;
    return 0;
}

cudaError_t launch_tc_iter(const IterLaunch& p, cudaStream_t st, int* launched) {
    *launched = 0;
    const Geom& g = p.g;
    const int split = iter_split(g);
    if (split == 0 || p.T < 1 || !p.tile_bits || !p.part || !p.gbar) return cudaErrorInvalidValue;
    CUtensorMap tmQ, tmK;
    const uint64_t rows = uint64_t(g.BH) * g.L;
    if (!tma_map_bf16(&tmQ, p.Q, rows, g.d, 128) || !tma_map_bf16(&tmK, p.K, rows, g.d, split == 1 ? 128 : 64))
        return cudaErrorInvalidValue;
    IterArgs a{};
    a.H = g.H;
    a.L = g.L;
    a.h = g.h;
    a.BH = g.BH;
    a.nst = g.L / 128;
    a.nw = iter_window_tiles(g.L, g.h);
    a.n_items = g.BH * a.nst;
    a.words = tile_words(g.L);
    a.sl2 = g.scale * kLog2e;
    a.logm = p.logm;
    a.tile_bits = p.tile_bits;
    a.u_tail = p.u_tail;
    a.v_tail = p.v_tail;
    a.pstride = p.pstride;
    a.vb2 = p.vb2;
    a.part = p.part;
    a.gbar = p.gbar;
    a.status = p.status;
    a.T = p.T;
    const int nk = p.T + p.R;
    if (p.fused) {
        a.k0 = 1;
        a.nk = nk;
        a.fused = 1;
        const cudaError_t e = g.d == 128 ? launch_iter_dh<128>(split, tmQ, tmK, a, st) : launch_iter_dh<64>(split, tmQ, tmK, a, st);
        if (e == cudaSuccess) *launched = 1;
        if (e == cudaSuccess || p.fused == 2) return e;
        (void)cudaGetLastError();   // a refused launch configuration: fall back to one launch per iteration
    }
    // one launch per iteration, then its column finalisation
    a.fused = 0;
    a.nk = 1;
    const long total = long(g.BH) * g.L;
    const int fgrid = int(std::min<long>((total + 255) / 256, 4L * sm_count()));
    for (int k = 1; k <= nk; ++k) {
        a.k0 = k;
        cudaError_t e = g.d == 128 ? launch_iter_dh<128>(split, tmQ, tmK, a, st) : launch_iter_dh<64>(split, tmQ, tmK, a, st);
        if (e != cudaSuccess) return e;
        finalize_kernel<<<fgrid, 256, 0, st>>>(a, k);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        *launched += 2;
    }
    return cudaSuccess;
}

}  // namespace eot
