// Tensor-core band sweeps for sm_100a: TMA tile loads into 128-byte-swizzled shared memory,
// tcgen05.mma (bf16 in, fp32 accumulate in TMEM) issued by one thread, warp-specialised
// roles, and register epilogues that read the score tiles back with tcgen05.ld.
//
// Method: "Blockwise Differentiable Sinkhorn Attention", technical summary (gist.science
// 2605.08123).  §2.1: each forward half-step is a band log-sum-exp
//     u_r = log a_r - LSE_{c in band(r)} (S_rc + v_c),   S = scale X Y^T,
// computed here with the previous potential as the shift (after a completed half-step every
// plan entry exp(S + u_old + v) is at most 1, so no running maximum is needed; the very
// first half-step of a call has no previous potential and keeps a running maximum).
// §2.2: the backward sweeps re-form the one reference plan P(R,R) per tile from S and the
// stored potentials, and apply the per-row / per-column orbit factors in registers.
//
// Two kernels:
//   tc_band_kernel   persistent, 128 x 128 score tiles, row reductions only (forward
//                    half-steps and the staircase sums of the backward pass)
//   tc_sweep_kernel  one CTA per 128-row tile, 128 x 128 score tiles, row reductions and a
//                    second MMA that multiplies coefficient tiles into d-wide outputs
//                    (forward output, dV, dQ, dK)
#include <cudaTypedefs.h>

#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"

namespace eot {

namespace {

constexpr float kNegInf = -__builtin_huge_valf();

// ---------------------------------------------------------------------------------------
// Host: TMA descriptors over a [rows, d] bf16 matrix, box {64 elements, box_rows}, 128B swizzle
// ---------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

bool make_map(CUtensorMap* m, const void* base, uint64_t rows, int d, int box_rows) {
    auto fn = encode_fn();
    if (!fn || !base || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
    cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(d) * 2};
    cuuint32_t box[2] = {64u, cuuint32_t(box_rows)};
    cuuint32_t es[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D TMA descriptor over a [rows, 16] bf16 matrix (the folded modifier operands), boxes of
// 16 x box_rows, 32-byte swizzle.
bool make_map_ext(CUtensorMap* m, const void* base, uint64_t rows, int box_rows) {
    auto fn = encode_fn();
    if (!fn || !base || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
    cuuint64_t dims[2] = {16u, cuuint64_t(rows)};
    cuuint64_t strides[1] = {32u};
    cuuint32_t box[2] = {16u, cuuint32_t(box_rows)};
    cuuint32_t es[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------------------
// Device: band tile list shared by all roles of a CTA
// ---------------------------------------------------------------------------------------
// Columns of tile width BN intersecting the band of rows [r0, r0 + BM) that hold at least
// one active band column (the dustbin position is excluded: its links are handled apart).
// Returns the number of tiles; tile column indices go to tiles[].  Also reports whether
// any row of the row tile is active.  Must be called by all threads.
template <int BM, int BN>
__device__ int build_tile_list(const float* logm, int L, int r0, int h, int D, int* tiles, int* flags,
                               int* ntiles_smem, bool* any_row) {
    const int tid = threadIdx.x;
    const int clo = max(0, r0 - h), chi = min(L - 1, r0 + BM - 1 + h);
    const int t_lo = clo / BN, t_hi = chi / BN;
    for (int t = tid; t <= t_hi - t_lo; t += blockDim.x) flags[t] = 0;
    __syncthreads();
    for (int c = clo + tid; c <= chi; c += blockDim.x)
        if (logm[c] != kNegInf && c != D) flags[c / BN - t_lo] = 1;
    int rowact = 0;
    for (int r = tid; r < BM; r += blockDim.x) rowact |= (logm[r0 + r] != kNegInf);
    const int any = __syncthreads_or(rowact);
    if (tid == 0) {
        int n = 0;
        for (int t = 0; t <= t_hi - t_lo; ++t)
            if (flags[t]) tiles[n++] = t_lo + t;
        *ntiles_smem = n;
    }
    __syncthreads();
    *any_row = any != 0;
    return *ntiles_smem;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ---------------------------------------------------------------------------------------
// Forward half-step (band log-sum-exp) and weighted band row sums: persistent kernel
// ---------------------------------------------------------------------------------------
// One CTA per SM walks a contiguous range of work items.  An item is a pair of adjacent
// 128-row tiles of one unit, rows [256 p, 256 p + 256); both halves share every 128-column
// tile that their bands touch, so each column tile comes into shared memory once and feeds
// two MMAs.  Roles:
//   warp 0       TMA producer (one lane): row halves into a small ring, column tiles into
//                NS stages, and per half the tile's column vectors (log2 bias, weights)
//   warp 1       TMEM allocator and MMA issuer of the first half (one lane); warp 2 issues
//                the second half's MMAs: two 128-column fp32 score accumulators per half
//                (4 x 128 TMEM columns).  One issue thread per half, because one thread's
//                per-MMA bookkeeping for both halves was slower than the tensor core.
//   warp 3       idle (it completes the first warpgroup)
//   warps 4..11  epilogue of the first half, warps 12..19 of the second: warp (q, hf) reads
//                TMEM lanes [32 q, 32 q + 32) of every other tile of its half (tiles whose
//                running index has parity hf, i.e. the tiles of TMEM buffer hf), all 128 columns,
//                so that a warp's per-tile waits and hand-backs are paid once per 128 columns
// Registers: the block is launched at 96 a thread; warpgroup 0 (warps 0-3) gives registers
// back (setmaxnreg 48) and the four epilogue warpgroups take them (104), so the epilogue's
// chain of score, exponential and sums keeps more values live (long workload, forward: 5.61 ->
// 5.33 ms against 96 registers everywhere; control warps at 40 or 56 registers: 5.43 / 5.36).
// The two warps that share a row meet once per item on a 64-thread named barrier; the
// halves are coupled only through the column-tile stages.  All roles walk the same item /
// tile sequence, so ring slots and mbarrier phases follow from running counters.
//
// Reductions (KIND), for the rows r of a half and the band columns c of each row:
//   online  out_r = logm_r - LSE_c (S_rc + colpot_c), with a running maximum (first step)
//   shift   the same sum shifted by the previous potential st_r: after a completed
//           half-step every term exp(S + st + colpot) is at most 1, so no maximum is kept
//   wsum    out_r = f_r hv_r sum_c exp(S_rc + st_r + colpot_c) w_c  (staircase sums of the
//           tail adjoint, with st = the row orbit bias and w = the column weights)
enum BandKind { kBandOnline = 0, kBandShift = 1, kBandWsum = 2 };

// Pairs of exponentials per 32-column chunk evaluated on the FMA pipe instead of MUFU in
// interior tiles of the band kernel (measured per half-step on the long workload: 0 pairs
// 0.2271 ms, 1 pair 0.2264, 2 pairs 0.2302, 3 pairs 0.2339).
constexpr int kFmaPairs = 1;

struct TcBandArgs {
    int H, L, h, D, n_items, items_per_cta, pairs_per_unit;
    float sl2;                  // scale * log2(e)
    float isl2;                 // 1 / sl2 (column-bias operand rows)
    const float* logm;
    const uint32_t* tile_bits;  // [B][words]: bit t = positions [128 t, 128 t + 128) hold an active non-dustbin token
    int words;
    const float* colbias2;      // [BH, L] masked log2 column bias
    const float* colw;          // [BH, L] column weights (wsum)
    const float* colpot;        // natural column potential (pstride), read at D
    const float* stab;          // natural row shift (pstride); unused by online
    float* out;                 // natural (pstride)
    float* out_bias2;           // [BH, L] masked log2 copy of out (log-sum-exp kinds)
    const float* f;             // [BH, L] row factors (wsum)
    const float* hv;            // [BH, L] (wsum)
    size_t pstride;
    const float* sd_term;
    uint32_t* status;
    // Several half-steps in one (cooperative) launch: half-steps hs0 .. hs0 + nhs - 1 of the
    // forward schedule (even: row, X = Q; odd: column, X = K; iteration hs / 2 updates slot 0
    // for the first T iterations and slot k = hs / 2 - T + 1 after), separated by a grid-wide
    // barrier (gbar[hs] counts the CTAs done with half-step hs).
    int hs0, nhs, T;
    float* u_tail;
    float* v_tail;
    float* ub2;
    float* vb2;
    uint32_t* gbar;
    // CTA c takes items [bounds[c], bounds[c + 1]) (schedule_kernel), or, when null, the
    // equal ranges of items_per_cta
    const int* bounds;
    // Fused half-steps with a dustbin: the dustbin links of the rows (sd_row: S between row r
    // and the dustbin column) and of the columns (sd_col: S between the dustbin row and column
    // c); the dense dustbin row of every half-step is summed per item ((max, sum) partials in
    // dpart[bh][pair]) and merged by the last item of the unit (dcnt[bh], zero at launch).
    const float* sd_row;
    const float* sd_col;
    float* dpart;
    uint32_t* dcnt;
    int dself;                  // (D, D) in the support
    const float* sadd;          // wsum: out_r = f_r (hv_r sum + sadd_r) when not null
    // Column-bias operand rows (see band_ext_row): written for every output position when not
    // null (a single half-step), and, in fused d = 128 half-steps, written and read through ue
    // (u side) and ve (v side), [BH L, 16] bf16 each.
    __nv_bfloat16* ext_out;
    __nv_bfloat16* ue;
    __nv_bfloat16* ve;
};

template <int DH, int KIND, bool EXT = false>
struct BandCfg {
    static constexpr int BM = 128, BN = 128;
    static constexpr int KATOMS = DH / 64;
    static constexpr int NQ = DH == 128 ? 3 : 6;   // row half-tile slots
    static constexpr int NS = DH == 128 ? 3 : 6;   // column-tile stages
    // column-vector slots per half (3 for the weighted sums with the bias in the product, whose
    // operand tiles take the room of the fourth)
    static constexpr int NV = (EXT && KIND == kBandWsum) ? 3 : 4;
    static constexpr int NVEC = KIND == kBandWsum ? 2 : 1;
    static constexpr uint32_t XB = BM * DH * 2;    // row half-tile bytes
    static constexpr uint32_t YB = BN * DH * 2;    // column tile bytes
    static constexpr uint32_t ATOM = 128 * 128;    // one 64-element-wide atom column of 128 rows
    static constexpr uint32_t VB = NVEC * BN * 4;  // column vectors of one tile
    static constexpr uint32_t OFF_Y = NQ * XB;
    static constexpr uint32_t OFF_V = OFF_Y + NS * YB;         // [half][NV][VB]
    static constexpr uint32_t OFF_RED = OFF_V + 2 * NV * VB;    // [half][parity][column half][m, s][128 rows]
    static constexpr uint32_t OFF_BITS = OFF_RED + 2 * 2 * 2 * 2 * 128 * 4;   // tile bits of the CTA's batch rows
    static constexpr int BITS_WORDS = 512;
    // column-bias operands (EXT): the constant row operand and one column operand per stage,
    // [128 x 16] bf16 each, 32-byte swizzled
    static constexpr uint32_t EXTB = 128 * 16 * 2;
    static constexpr uint32_t OFF_ONES = (OFF_BITS + BITS_WORDS * 4 + 1023) / 1024 * 1024;
    static constexpr uint32_t OFF_YE = OFF_ONES + EXTB;
    static constexpr uint32_t OFF_BAR = EXT ? OFF_YE + NS * EXTB : OFF_BITS + BITS_WORDS * 4;
    // full[NS] empty[NS] qfull[NQ] qempty[NQ], then per half: tfull[2] tempty[2] vfull[NV] vempty[NV]
    static constexpr uint32_t HB0 = 2 * NS + 2 * NQ;
    static constexpr uint32_t HBN = 4 + 2 * NV;
    static constexpr uint32_t NBARS = HB0 + 2 * HBN;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr size_t SMEM = 1024 + OFF_MISC + 64;
    static_assert(SMEM <= 227 * 1024, "band kernel shared memory");
    static constexpr uint32_t IDESC = ptx::idesc_bf16(128, 128, false, false);
};

constexpr int kBandThreads = 640;   // TMA warp, MMA warps (halves 0, 1), an idle warp, 16 epilogue warps
constexpr int kBandIssuerB = 2;
constexpr int kBandEpi0 = 4;
constexpr int kBandLaunchRegs = 96;

// Decoded work item: rows [r0, r0 + 256) of unit bh as two halves with their column-tile bands.
struct BandItem {
    int bh, b, r0;
    size_t base;
    bool exists[2], active[2];
    int t_lo[2], t_hi[2];
};

__device__ __forceinline__ bool tile_bit(const uint32_t* bits, int t) { return (bits[t >> 5] >> (t & 31)) & 1u; }

// Tile bits of one batch row, the current 32-bit word held in a register.
struct TileBits {
    const uint32_t* w;
    int idx;
    uint32_t word;
    __device__ explicit TileBits(const uint32_t* p) : w(p), idx(-1), word(0u) {}
    __device__ bool operator()(int t) {
        if ((t >> 5) != idx) {
            idx = t >> 5;
            word = w[idx];
        }
        return (word >> (t & 31)) & 1u;
    }
};

// EXT (fused d = 128 half-steps of a wide band): the column bias comes out of the score product
// (band_ext_row).  Its operand rows are written in the previous half-step, so the first product
// of a half-step waits for the grid-wide barrier; with a short band (few tiles a row) that wait
// costs more than the fold saves (protein-like workload, W = 128: 3.12 -> 3.28 ms per call), so
// the launch selects it for W >= 512 only (long workload: 7.85 -> 7.70 ms).
template <int DH, int KIND, bool MULTI, bool EXT>
__global__ void __launch_bounds__(kBandThreads, 1)
    tc_band_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                   const __grid_constant__ CUtensorMap tmUE, const __grid_constant__ CUtensorMap tmVE,
                   const TcBandArgs a) {
    static_assert(!EXT || (DH == 128 && ((MULTI && KIND == kBandShift) || (!MULTI && KIND == kBandWsum))),
                  "the folded column bias is a d = 128 form of the fused half-steps and of the weighted sums");
    using C = BandCfg<DH, KIND, EXT>;
    constexpr bool ONLINE = KIND == kBandOnline, WSUM = KIND == kBandWsum;
    // column vectors: none with the bias in the product, except the weights of a weighted sum
    constexpr bool NOVEC = EXT && !WSUM;
    static_assert(!MULTI || KIND == kBandShift, "fused half-steps are shifted log-sum-exp sweeps");
    // Operands of half-step hs (a single launch uses the fixed pointers of a).
    const int hs_end = a.hs0 + a.nhs;
    auto slot_of = [&](int hs, bool out) {
        const int it = hs >> 1;
        return it < a.T ? 0 : (out ? it - a.T + 1 : it - a.T);
    };
    auto colbias_of = [&](int hs) -> const float* { return MULTI ? ((hs & 1) ? a.ub2 : a.vb2) : a.colbias2; };
    auto stab_of = [&](int hs) -> const float* {
        return MULTI ? ((hs & 1) ? a.v_tail : a.u_tail) + size_t(slot_of(hs, false)) * a.L : a.stab;
    };
    auto out_of = [&](int hs) -> float* {
        return MULTI ? ((hs & 1) ? a.v_tail : a.u_tail) + size_t(slot_of(hs, true)) * a.L : a.out;
    };
    auto outb_of = [&](int hs) -> float* { return MULTI ? ((hs & 1) ? a.vb2 : a.ub2) : a.out_bias2; };
    // column-bias operand rows written by half-step hs (and, EXT, read by it: the other side's)
    auto exto_of = [&](int hs) -> __nv_bfloat16* {
        return MULTI ? (EXT ? ((hs & 1) ? a.ve : a.ue) : nullptr) : a.ext_out;
    };
    // natural column potential (read at the dustbin) and the rows' dustbin links
    auto colpot_of = [&](int hs) -> const float* {
        return MULTI ? ((hs & 1) ? a.u_tail + size_t(slot_of(hs, true)) * a.L : a.v_tail + size_t(slot_of(hs, false)) * a.L)
                     : a.colpot;
    };
    auto sdterm_of = [&](int hs) -> const float* { return MULTI ? ((hs & 1) ? a.sd_col : a.sd_row) : a.sd_term; };
    auto mapx_of = [&](int hs) { return (MULTI && (hs & 1)) ? &tmY : &tmX; };
    auto mapy_of = [&](int hs) { return (MULTI && (hs & 1)) ? &tmX : &tmY; };
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = align1024(smraw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.L, h = a.h, D = a.D;
    const int item0 = a.bounds ? a.bounds[blockIdx.x] : blockIdx.x * a.items_per_cta;
    const int item1 = a.bounds ? a.bounds[blockIdx.x + 1] : min(a.n_items, item0 + a.items_per_cta);

    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    const uint32_t bar0 = ptx::smem_u32(bars);
    auto full = [&](int i) { return bar0 + 8u * i; };
    auto empty = [&](int i) { return bar0 + 8u * (C::NS + i); };
    auto qfull = [&](int i) { return bar0 + 8u * (2 * C::NS + i); };
    auto qempty = [&](int i) { return bar0 + 8u * (2 * C::NS + C::NQ + i); };
    auto tfull = [&](int G, int i) { return bar0 + 8u * (C::HB0 + G * C::HBN + i); };
    auto tempty = [&](int G, int i) { return bar0 + 8u * (C::HB0 + G * C::HBN + 2 + i); };
    auto vfull = [&](int G, int i) { return bar0 + 8u * (C::HB0 + G * C::HBN + 4 + i); };
    auto vempty = [&](int G, int i) { return bar0 + 8u * (C::HB0 + G * C::HBN + 4 + C::NV + i); };
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    // The tile bits of the batch rows this CTA's items touch, copied into shared memory when
    // they fit (every role reads them for every item and tile).
    uint32_t* sbits = reinterpret_cast<uint32_t*>(sm + C::OFF_BITS);
    const int b_first = item1 > item0 ? (item0 / a.pairs_per_unit) / a.H : 0;
    const int b_last = item1 > item0 ? ((item1 - 1) / a.pairs_per_unit) / a.H : -1;
    const int nbw = (b_last - b_first + 1) * a.words;
    const bool bits_in_smem = nbw <= C::BITS_WORDS;
    if (bits_in_smem)
        for (int i = tid; i < nbw; i += blockDim.x) sbits[i] = a.tile_bits[size_t(b_first) * a.words + i];
    const uint32_t* bits0 = bits_in_smem ? sbits : a.tile_bits + size_t(b_first) * a.words;
    auto bits_of = [&](int b) -> const uint32_t* { return bits0 + (b - b_first) * a.words; };

    auto decode = [&](int item) {
        BandItem it;
        it.bh = item / a.pairs_per_unit;
        it.b = it.bh / a.H;
        it.r0 = (item - it.bh * a.pairs_per_unit) * 2 * C::BM;
        it.base = size_t(it.bh) * L;
        const uint32_t* bits = bits_of(it.b);
#pragma unroll
        for (int G = 0; G < 2; ++G) {
            const int rg = it.r0 + G * C::BM;
            it.exists[G] = rg < L;
            it.active[G] = it.exists[G] && tile_bit(bits, rg / C::BM);
            it.t_lo[G] = max(0, rg - h) / C::BN;
            it.t_hi[G] = min(L - 1, rg + C::BM - 1 + h) / C::BN;
        }
        return it;
    };
    // Column tiles that half G multiplies: inside its band and holding an active column.
    auto uses = [&](const BandItem& it, int G, int t) { return it.active[G] && t >= it.t_lo[G] && t <= it.t_hi[G]; };

    if (EXT) {
        // constant row operand: logical 16-byte chunk 0 of every row is (1, 1, 1, 0, 0, 0, 0, 0),
        // chunk 1 zeros; the 32-byte swizzle stores chunk c of row r at c ^ ((r >> 2) & 1)
        uint32_t* ones = reinterpret_cast<uint32_t*>(sm + C::OFF_ONES);
        for (int i = tid; i < 128 * 8; i += blockDim.x) {
            const int r = i >> 3, pc = (i >> 2) & 1, w = i & 3;
            const int lc = pc ^ ((r >> 2) & 1);
            ones[i] = lc == 0 ? (w == 0 ? 0x3f803f80u : w == 1 ? 0x00003f80u : 0u) : 0u;
        }
        ptx::fence_proxy_async_smem();
    }
    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < C::NS; ++i) { ptx::mbar_init(full(i), 1); ptx::mbar_init(empty(i), 2); }
        for (int i = 0; i < C::NQ; ++i) { ptx::mbar_init(qfull(i), 1); ptx::mbar_init(qempty(i), 1); }
        for (int G = 0; G < 2; ++G) {
            // a score buffer and a column-vector slot are read by the four quadrant warps of one
            // column half (tiles alternate between the halves)
            for (int i = 0; i < 2; ++i) { ptx::mbar_init(tfull(G, i), 1); ptx::mbar_init(tempty(G, i), 4); }
            for (int i = 0; i < C::NV; ++i) { ptx::mbar_init(vfull(G, i), 1); ptx::mbar_init(vempty(G, i), 4); }
        }
        ptx::mbar_fence_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(misc), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tbase = misc[0];

    if (warp < kBandEpi0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 48;");
    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            ptx::prefetch_tmap(&tmX);
            ptx::prefetch_tmap(&tmY);
            if (EXT) {
                ptx::prefetch_tmap(&tmUE);
                ptx::prefetch_tmap(&tmVE);
            }
            int g = 0, qi = 0;
            int gv[2] = {0, 0};
            bool ok = true;
            for (int hs = a.hs0; hs < hs_end && ok; ++hs) {
            const CUtensorMap* mX = mapx_of(hs);
            const CUtensorMap* mY = mapy_of(hs);
            const float* cb2 = colbias_of(hs);
            // the column biases of half-step hs are written by every CTA in half-step hs - 1
            bool biases_ready = !MULTI || hs == a.hs0;
            for (int item = item0; item < item1 && ok; ++item) {
                const BandItem it = decode(item);
                if (!it.active[0] && !it.active[1]) continue;
#pragma unroll
                for (int G = 0; G < 2; ++G) {
                    if (!it.active[G]) continue;
                    const int qb = qi % C::NQ;
                    if (!ptx::mbar_wait(qempty(qb), ((qi / C::NQ) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                    ptx::mbar_expect_tx(qfull(qb), C::XB);
                    const uint32_t xs = ptx::smem_u32(sm + qb * C::XB);
                    for (int ka = 0; ka < C::KATOMS; ++ka)
                        ptx::tma_load_2d(xs + ka * C::ATOM, mX, ka * 64, int(it.base) + it.r0 + G * C::BM, qfull(qb));
                    ++qi;
                }
                if (!ok) break;
                TileBits bits(bits_of(it.b));
                const int u_lo = it.active[0] ? it.t_lo[0] : it.t_lo[1];
                const int u_hi = it.active[1] ? it.t_hi[1] : it.t_hi[0];
                for (int t = u_lo; t <= u_hi && ok; ++t) {
                    if (!bits(t)) continue;
                    const bool use0 = uses(it, 0, t), use1 = uses(it, 1, t);
                    if (!use0 && !use1) continue;
                    const int c0 = t * C::BN;
                    const int s = g % C::NS;
                    if (!ptx::mbar_wait(empty(s), ((g / C::NS) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                    ptx::mbar_expect_tx(full(s), C::YB + (EXT ? C::EXTB : 0u));
                    const uint32_t ys = ptx::smem_u32(sm + C::OFF_Y + s * C::YB);
                    for (int ka = 0; ka < C::KATOMS; ++ka)
                        ptx::tma_load_2d(ys + ka * C::ATOM, mY, ka * 64, int(it.base) + c0, full(s));
                    ++g;
                    if (!biases_ready) {
                        if (!ptx::grid_wait(a.gbar + hs - 1, gridDim.x, abort_flag, a.status)) {
                            // the stage still expects its column-bias operand: fill it so that
                            // no copy is left pending when the CTA retires
                            if (EXT)
                                ptx::tma_load_2d(ptx::smem_u32(sm + C::OFF_YE + s * C::EXTB), (MULTI && !(hs & 1)) ? &tmVE : &tmUE, 0,
                                                 int(it.base) + c0, full(s));
                            ok = false;
                            break;
                        }
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                        biases_ready = true;
                    }
                    // the column-bias operand rows of half-step hs were written in half-step hs - 1
                    if (EXT)
                        ptx::tma_load_2d(ptx::smem_u32(sm + C::OFF_YE + s * C::EXTB), (MULTI && !(hs & 1)) ? &tmVE : &tmUE, 0,
                                         int(it.base) + c0, full(s));
                    // (with the column bias in the product the epilogue reads no column vectors)
#pragma unroll
                    for (int G = 0; G < 2; ++G) {
                        if (NOVEC || !(G ? use1 : use0)) continue;
                        const int vs = gv[G] % C::NV;
                        if (!ptx::mbar_wait(vempty(G, vs), ((gv[G] / C::NV) & 1) ^ 1, abort_flag, a.status)) {
                            ok = false;
                            break;
                        }
                        ptx::mbar_expect_tx(vfull(G, vs), C::VB);
                        const uint32_t vd = ptx::smem_u32(sm + C::OFF_V + (G * C::NV + vs) * C::VB);
                        ptx::bulk_load(vd, cb2 + it.base + c0, C::BN * 4, vfull(G, vs));
                        if (WSUM) ptx::bulk_load(vd + C::BN * 4, a.colw + it.base + c0, C::BN * 4, vfull(G, vs));
                        ++gv[G];
                    }
                }
            }
            }
            if (*abort_flag) {
                // Let every copy already issued land before the CTA retires.
                volatile int dummy = 0;
                for (int i = max(0, g - C::NS); i < g; ++i) ptx::mbar_wait(full(i % C::NS), (i / C::NS) & 1, &dummy, a.status);
                for (int G = 0; G < 2; ++G)
                    for (int i = max(0, gv[G] - C::NV); i < gv[G]; ++i)
                        ptx::mbar_wait(vfull(G, i % C::NV), (i / C::NV) & 1, &dummy, a.status);
                for (int i = max(0, qi - C::NQ); i < qi; ++i) ptx::mbar_wait(qfull(i % C::NQ), (i / C::NQ) & 1, &dummy, a.status);
            }
        }
    } else if (warp == 1 || warp == kBandIssuerB) {
        if (lane == 0) {
            // ---------------- MMA issuers: warp 1 for row half 0, warp kBandIssuerB for half 1 ----------------
            // Two issuing threads halve the per-instruction bookkeeping each one carries; both
            // walk every column tile (a stage is free once both have committed it).
            const int GI = warp == 1 ? 0 : 1;
            int g = 0, qi = 0, gt = 0;
            bool ok = true;
            for (int hs = a.hs0; hs < hs_end && ok; ++hs)
            for (int item = item0; item < item1 && ok; ++item) {
                const BandItem it = decode(item);
                if (!it.active[0] && !it.active[1]) continue;
                TileBits bits(bits_of(it.b));
                int qslot = 0, qpar = 0, n = 0, done = 0;
                bool xready = false;
#pragma unroll
                for (int G = 0; G < 2; ++G) {
                    if (!it.active[G]) continue;
                    if (G == GI) {
                        qslot = qi % C::NQ;
                        qpar = (qi / C::NQ) & 1;
                        for (int t = it.t_lo[G]; t <= it.t_hi[G]; ++t) n += bits(t);
                    }
                    ++qi;
                }
                const bool mine = it.active[GI];
                const int u_lo = it.active[0] ? it.t_lo[0] : it.t_lo[1];
                const int u_hi = it.active[1] ? it.t_hi[1] : it.t_hi[0];
                for (int t = u_lo; t <= u_hi && ok; ++t) {
                    if (!bits(t)) continue;
                    const bool use0 = uses(it, 0, t), use1 = uses(it, 1, t);
                    if (!use0 && !use1) continue;
                    const int s = g % C::NS;
                    // the stage's current fill must have landed before this thread's commit on it counts
                    if (!ptx::mbar_wait(full(s), (g / C::NS) & 1, abort_flag, a.status)) { ok = false; break; }
                    if (GI ? use1 : use0) {
                        if (!xready) {
                            if (!ptx::mbar_wait(qfull(qslot), qpar, abort_flag, a.status)) { ok = false; break; }
                            xready = true;
                        }
                        const int tb = gt & 1;
                        if (!ptx::mbar_wait(tempty(GI, tb), ((gt >> 1) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                        ptx::tc_fence_after();
                        // descriptor start addresses advance in 16-byte units within one field
                        const uint64_t xd = ptx::smem_desc(ptx::smem_u32(sm + qslot * C::XB), 16, 1024);
                        const uint64_t yd = ptx::smem_desc(ptx::smem_u32(sm + C::OFF_Y + s * C::YB), 16, 1024);
                        const uint32_t dt = tbase + uint32_t((GI * 2 + tb) * C::BN);
#pragma unroll
                        for (int kk = 0; kk < DH / 16; ++kk) {
                            const uint64_t koff = uint64_t(((kk >> 2) * C::ATOM + (kk & 3) * 32) >> 4);
                            ptx::mma_bf16(dt, xd + koff, yd + koff, C::IDESC, kk > 0 ? 1u : 0u);
                        }
                        // + the column bias b_c / (scale log2 e) (band_ext_row)
                        if (EXT)
                            ptx::mma_bf16(dt, ptx::smem_desc_sw32(ptx::smem_u32(sm + C::OFF_ONES)),
                                          ptx::smem_desc_sw32(ptx::smem_u32(sm + C::OFF_YE + s * C::EXTB)), C::IDESC, 1u);
                        ptx::mma_commit(tfull(GI, tb));
                        ++gt;
                        if (++done == n) ptx::mma_commit(qempty(qslot));   // row half free once its products are done
                    }
                    ptx::mma_commit(empty(s));
                    ++g;
                }
                // (a half with no column tile cannot occur: an active row tile holds its own diagonal tile)
                if (ok && mine && n == 0) {
                    if (!ptx::mbar_wait(qfull(qslot), qpar, abort_flag, a.status)) ok = false;
                    else ptx::mma_commit(qempty(qslot));
                }
            }
            if (*abort_flag && gt > 0) {
                volatile int dummy = 0;
                ptx::mbar_wait(tfull(GI, (gt - 1) & 1), ((gt - 1) >> 1) & 1, &dummy, a.status);
            }
        }
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 104;");
        // ---------------- epilogue: 8 warps per half ----------------
        const int e = warp - kBandEpi0;
        const int G = e >> 3;                 // row half
        const int hf = (e >> 2) & 1;          // column half of each tile
        const int q = warp & 3;               // TMEM lane quadrant (fixed by the warp's rank)
        const int row = q * 32 + lane;
        const uint32_t lane_base = uint32_t(q * 32) << 16;
        float* red = reinterpret_cast<float*>(sm + C::OFF_RED) + G * (2 * 2 * 2 * 128);
        const uint32_t vsm = ptx::smem_u32(sm + C::OFF_V + G * C::NV * C::VB);
        int gt = 0, ep = 0;
        bool ok = true;
        for (int hs = a.hs0; hs < hs_end; ++hs) {
        const float* stab_hs = stab_of(hs);
        float* out_hs = out_of(hs);
        float* outb_hs = outb_of(hs);
        if (MULTI && hs > a.hs0) {
            // every CTA has written half-step hs - 1 (the shifts and biases read below)
            if (tid == 32 * kBandEpi0 && ok && !ptx::grid_wait(a.gbar + hs - 1, gridDim.x, abort_flag, a.status)) ok = false;
            ptx::named_bar_sync(9, 512);
            ok = ok && !*abort_flag;
        }
        for (int item = item0; item < item1; ++item) {
            // this half of the item (no per-half arrays: G is not a compile-time index here)
            const int bh = item / a.pairs_per_unit, b = bh / a.H;
            const int rg = (item - bh * a.pairs_per_unit) * 2 * C::BM + G * C::BM;
            if (rg >= L) continue;
            const size_t base = size_t(bh) * L;
            const int r = rg + row;
            const size_t pb = size_t(bh) * a.pstride;
            const uint32_t* bitp = bits_of(b);
            if (!tile_bit(bitp, rg / C::BM)) {
                // (fused half-steps: an active dustbin's row is written by the dense dustbin row;
                // a single half-step's dense dustbin kernel runs after this one)
                if (hf == 0 && !(MULTI && r == D && a.logm[size_t(b) * L + D] != kNegInf)) {
                    out_hs[pb + r] = 0.f;
                    if (!WSUM) outb_hs[base + r] = kNegInf;
                }
                if (!WSUM && hf == 0 && exto_of(hs)) band_ext_row(exto_of(hs) + (base + r) * 16, kNegInf, a.isl2);
                continue;
            }
            const int t_lo = max(0, rg - h) / C::BN, t_hi = min(L - 1, rg + C::BM - 1 + h) / C::BN;
            const float* logm = a.logm + size_t(b) * L;
            const float lm = logm[r];
            const float st = ONLINE ? 0.f : stab_hs[pb + r];
            const float st2 = st * kLog2e;
            float m_run = kNegInf;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            TileBits bits(bitp);
            // One 32-column chunk starting at column cc: scores v -> partial sums.  The chunk's
            // column bias (and weights) sit in shared memory at vaddr (and vaddr + 4 BN).
            // masked: some entries of the chunk lie outside the band of their row.
            auto process = [&](const float (&v)[32], int cc, uint32_t vaddr, bool masked) {
                if (ONLINE || masked) {
                    float x[32];
                    if (EXT) {
                        // the accumulator holds S + b_c / (scale log2 e): x = exponent incl. the shift
#pragma unroll
                        for (int j = 0; j < 32; ++j) x[j] = fmaf(v[j], a.sl2, st2);
                    } else {
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 bv = ptx::ld_shared_f4(vaddr + 16u * j4);
                            x[4 * j4 + 0] = fmaf(v[4 * j4 + 0], a.sl2, bv.x);
                            x[4 * j4 + 1] = fmaf(v[4 * j4 + 1], a.sl2, bv.y);
                            x[4 * j4 + 2] = fmaf(v[4 * j4 + 2], a.sl2, bv.z);
                            x[4 * j4 + 3] = fmaf(v[4 * j4 + 3], a.sl2, bv.w);
                        }
                    }
                    if (masked) {
                        // valid columns j of this chunk: r - h <= cc + j <= r + h
                        const int lo = r - h - cc, hi = r + h - cc;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (j < lo || j > hi) x[j] = kNegInf;
                    }
                    if (ONLINE) {
                        float cm = kNegInf;
#pragma unroll
                        for (int j = 0; j < 32; ++j) cm = fmaxf(cm, x[j]);
                        if (cm > m_run) {
                            const float sc = ptx::ex2(m_run - cm);
#pragma unroll
                            for (int k = 0; k < 4; ++k) acc[k] *= sc;
                            m_run = cm;
                        }
                        if (m_run != kNegInf) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) acc[j & 3] += ptx::ex2(x[j] - m_run);
                        }
                    } else if (WSUM) {
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 wv = ptx::ld_shared_f4(vaddr + 4u * C::BN + 16u * j4);
                            // (with the bias in the product, x already holds the shift)
                            const float sh = EXT ? 0.f : st2;
                            acc[0] = fmaf(ptx::ex2(x[4 * j4 + 0] + sh), wv.x, acc[0]);
                            acc[1] = fmaf(ptx::ex2(x[4 * j4 + 1] + sh), wv.y, acc[1]);
                            acc[2] = fmaf(ptx::ex2(x[4 * j4 + 2] + sh), wv.z, acc[2]);
                            acc[3] = fmaf(ptx::ex2(x[4 * j4 + 3] + sh), wv.w, acc[3]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) acc[j & 3] += ptx::ex2(EXT ? x[j] : x[j] + st2);
                    }
                } else {
                    // every entry inside the band, shifted: packed fp32x2 math
                    const uint64_t SL2 = ptx::f2(a.sl2, a.sl2), ST2 = ptx::f2(st2, st2);
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4) {
                        float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (!EXT) bv = ptx::ld_shared_f4(vaddr + 16u * j4);
                        float4 wv;
                        if (WSUM) wv = ptx::ld_shared_f4(vaddr + 4u * C::BN + 16u * j4);
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int k = 2 * j4 + hh;
                            uint64_t xx;
                            if (EXT) {
                                // bias already in the accumulator: one packed FMA with the row shift
                                xx = ptx::ffma2(ptx::f2(v[2 * k], v[2 * k + 1]), SL2, ST2);
                            } else {
                                xx = ptx::ffma2(ptx::f2(v[2 * k], v[2 * k + 1]), SL2,
                                                hh ? ptx::f2(bv.z, bv.w) : ptx::f2(bv.x, bv.y));
                                xx = ptx::fadd2(xx, ST2);
                            }
                            float x0, x1, e0, e1;
                            ptx::f2split(xx, x0, x1);
                            if (k < kFmaPairs) {
                                ptx::exp2_fma_x2(x0, x1, e0, e1);
                            } else {
                                e0 = ptx::ex2(x0);
                                e1 = ptx::ex2(x1);
                            }
                            // the pair's two fp32 sums in one packed instruction
                            float* ap = acc + 2 * hh;
                            if (WSUM)
                                ptx::f2split(ptx::ffma2(ptx::f2(e0, e1), hh ? ptx::f2(wv.z, wv.w) : ptx::f2(wv.x, wv.y),
                                                        ptx::f2(ap[0], ap[1])), ap[0], ap[1]);
                            else
                                ptx::f2split(ptx::fadd2(ptx::f2(ap[0], ap[1]), ptx::f2(e0, e1)), ap[0], ap[1]);
                        }
                    }
                }
            };
            // Band position of a 32 x 32 block (this warp's rows, one 32-column chunk): 0 =
            // outside the band for every row (skipped: no TMEM read, no exponentials),
            // 1 = inside for every entry, 2 = cut by the band edge (masked per entry).
            const int rw = rg + q * 32;
            auto block_class = [&](int cc) {
                const int dmin = cc - (rw + 31), dmax = cc + 31 - rw;   // range of c - r
                if (dmin > h || dmax < -h) return 0;
                return (dmax <= h && dmin >= -h) ? 1 : 2;
            };
            for (int t = t_lo; t <= t_hi; ++t) {
                if (!bits(t)) continue;
                const int gg = gt++;
                // the two column-half warps of a quadrant take alternate tiles (the tile's parity
                // is also its TMEM buffer), all 128 columns each
                if ((gg & 1) != hf || !ok) continue;
                const int c0 = t * C::BN;
                const int tb = gg & 1, vs = gg % C::NV;
                // Waits are made warp-uniform: the tcgen05.ld below is a warp-collective (.aligned).
                bool w1 = NOVEC || ptx::mbar_wait(vfull(G, vs), (gg / C::NV) & 1, abort_flag, a.status);
                bool w2 = w1 && ptx::mbar_wait(tfull(G, tb), (gg >> 1) & 1, abort_flag, a.status);
                if (!__all_sync(0xffffffffu, w2)) { ok = false; continue; }
                ptx::tc_fence_after();
                const uint32_t vaddr = vsm + uint32_t(vs) * C::VB;
                const uint32_t tcol = tbase + lane_base + uint32_t((G * 2 + tb) * C::BN);
                int last_k = -1;   // the last 32-column chunk with a score read
                for (int k = 0; k < 4; ++k)
                    if (block_class(c0 + 32 * k) != 0) last_k = k;
#pragma unroll 1
                for (int k = 0; k < 4; ++k) {
                    const int cc = c0 + 32 * k, kc = block_class(cc);
                    if (kc == 0) continue;
                    float v[32];
                    ptx::tmem_ld32(tcol + uint32_t(32 * k), v);
                    ptx::tmem_wait_ld(v);
                    if (k == last_k) {
                        // this warp's part of the accumulator is read: hand it back
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(tempty(G, tb));
                    }
                    process(v, cc, vaddr + 128u * uint32_t(k), kc == 2);
                }
                if (last_k < 0) {
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(tempty(G, tb));
                }
                __syncwarp();
                if (!NOVEC && lane == 0) ptx::mbar_arrive(vempty(G, vs));
            }
            // The two column halves of each row meet in shared memory (two parity slots: the
            // partner writes item e + 2 only after this warp has read item e).  Both warps form
            // the same total (half 0's partial first), then half 0 writes the potential and its
            // log2 copy and half 1 the column-bias operand row.
            float* rd = red + (ep & 1) * (2 * 2 * 128);
            ++ep;
            const float part = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            rd[hf * 256 + row] = m_run;
            rd[hf * 256 + 128 + row] = part;
            ptx::named_bar_sync(1 + G * 4 + q, 64);
            const bool is_dustbin_row = (r == D) && lm != kNegInf;
            const bool writes_ext = !WSUM && exto_of(hs) != nullptr;
            if ((hf == 0 || writes_ext) && ok && !*abort_flag && !is_dustbin_row) {
                const float m1 = rd[(1 - hf) * 256 + row], s1 = rd[(1 - hf) * 256 + 128 + row];
                float mm = hf == 0 ? m_run : m1, sum = hf == 0 ? part : s1;
                const float mo = hf == 0 ? m1 : m_run, so = hf == 0 ? s1 : part;
                if (ONLINE) lse2_merge(mm, sum, mo, so);
                else sum += so;
                float outv = 0.f, ob = kNegInf;
                if (lm != kNegInf) {
                    const bool d_act = D >= 0 && logm[D] != kNegInf;
                    if (ONLINE) {
                        if (d_act) lse2_add(mm, sum, (sdterm_of(hs)[base + r] + colpot_of(hs)[pb + D]) * kLog2e);
                        outv = lm - (mm + ptx::lg2(sum)) * kLn2;
                    } else {
                        const float dterm =
                            d_act ? ptx::ex2((sdterm_of(hs)[base + r] + colpot_of(hs)[pb + D]) * kLog2e + st2) : 0.f;
                        if (WSUM) {
                            if (d_act) sum = fmaf(dterm, a.colw[base + D], sum);
                            outv = a.f[base + r] * (a.hv[base + r] * sum + (a.sadd ? a.sadd[base + r] : 0.f));
                        } else {
                            outv = lm - ptx::lg2(sum + dterm) * kLn2 + st;
                        }
                    }
                    if (hf == 0 && !isfinite(outv)) atomicOr(a.status, kStatusNonFinite);
                    ob = outv * kLog2e;
                }
                if (hf == 0) {
                    out_hs[pb + r] = outv;
                    if (!WSUM) outb_hs[base + r] = ob;
                } else {
                    band_ext_row(exto_of(hs) + (base + r) * 16, ob, a.isl2);
                }
            } else if (writes_ext && hf == 1 && is_dustbin_row) {
                band_ext_row(exto_of(hs) + (base + r) * 16, kNegInf, a.isl2);   // the dustbin never enters a band sum
            }
        }
        if (MULTI && D >= 0 && __all_sync(0xffffffffu, ok && !*abort_flag)) {
            // Dense dustbin row of half-step hs: out_D = logm_D - LSE_c (S_Dc + colpot_c) over
            // every active real column c (plus (D, D) when it is in the support).  Epilogue warp e
            // sums the columns of this CTA's items e, e + 16, ... (the item's 256 positions); the
            // last item of a unit to finish merges the unit's partials.
            const float* colpot_hs = colpot_of(hs);
            const float* sdterm_hs = sdterm_of(hs);
            for (int item = item0 + e; item < item1; item += 16) {
                const int bh = item / a.pairs_per_unit, b = bh / a.H, pi = item - bh * a.pairs_per_unit;
                const float* logm = a.logm + size_t(b) * L;
                if (logm[D] == kNegInf) continue;
                const size_t base = size_t(bh) * L, pb = size_t(bh) * a.pstride;
                const float* sdense = (hs & 1) ? a.sd_row : a.sd_col;
                float m = kNegInf, s = 0.f;
                const int c_end = min(L, pi * 2 * C::BM + 2 * C::BM);
                for (int c = pi * 2 * C::BM + lane; c < c_end; c += 32) {
                    if (c == D) {
                        if (a.dself) lse2_add(m, s, (sdterm_hs[base + D] + colpot_hs[pb + D]) * kLog2e);
                    } else if (logm[c] != kNegInf) {
                        lse2_add(m, s, (sdense[base + c] + colpot_hs[pb + c]) * kLog2e);
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float m2 = __shfl_xor_sync(0xffffffffu, m, off), s2 = __shfl_xor_sync(0xffffffffu, s, off);
                    lse2_merge(m, s, m2, s2);
                }
                float* part = a.dpart + size_t(bh) * 2 * a.pairs_per_unit;
                uint32_t last = 0;
                if (lane == 0) {
                    part[2 * pi] = m;
                    part[2 * pi + 1] = s;
                    __threadfence();
                    last = atomicAdd(a.dcnt + bh, 1u) == uint32_t(a.pairs_per_unit - 1);
                }
                if (!__shfl_sync(0xffffffffu, last, 0)) continue;
                __threadfence();
                float mm = kNegInf, ss = 0.f;
                for (int i = lane; i < a.pairs_per_unit; i += 32) lse2_merge(mm, ss, __ldcg(part + 2 * i), __ldcg(part + 2 * i + 1));
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float m2 = __shfl_xor_sync(0xffffffffu, mm, off), s2 = __shfl_xor_sync(0xffffffffu, ss, off);
                    lse2_merge(mm, ss, m2, s2);
                }
                if (lane == 0) {
                    const float outv = logm[D] - (mm + log2f(ss)) * kLn2;
                    if (!isfinite(outv)) atomicOr(a.status, kStatusNonFinite);
                    out_hs[pb + D] = outv;
                    outb_hs[base + D] = kNegInf;   // the dustbin never enters a band sum
                    a.dcnt[bh] = 0u;                 // ready for the next half-step
                }
            }
        }
        if (MULTI) {
            // this CTA is done with half-step hs: count it on the grid-wide barrier
            ptx::named_bar_sync(9, 512);
            if (tid == 32 * kBandEpi0) {
                __threadfence();
                asm volatile("fence.proxy.async.global;" ::: "memory");
                atomicAdd(a.gbar + hs, 1u);
            }
        }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tbase, 512);
    }
}

// ---------------------------------------------------------------------------------------
// Output / backward sweep, 128 x 128 tiles
// ---------------------------------------------------------------------------------------
// Pass kinds (compile-time, so that each variant carries only its own arithmetic):
//   Out    O  = sum_c (P/a)_rc V_c                                   (forward output)
//   C1     beta_R = sum_c Pt_rc dP_rc  and  dV = sum_c Pt_rc dO_c     (column sweep)
//   R2     alpha_R = sum_c Pt dP + hv_r sum_c Pt m_c                  (row sweep)
//   Stair  f_r * hv_r * sum_c P_rc m_c   (staircase sweeps; run as weighted band sums by tc_band_kernel)
//   Grad   dQ / dK = scale sum_c Pt_rc (dP_rc - sum_k xr_k yc_k) Y_c  (final sweeps)
enum SweepMode { kModeOut = 0, kModeC1 = 1, kModeR2 = 2, kModeStair = 3, kModeGrad = 4 };

template <int MODE>
struct ModeT {
    static constexpr bool SCAL = MODE == kModeC1 || MODE == kModeR2 || MODE == kModeStair;
    static constexpr bool SDP = MODE == kModeC1 || MODE == kModeR2;
    static constexpr bool SM = MODE == kModeR2 || MODE == kModeStair;
    static constexpr bool VEC = MODE == kModeOut || MODE == kModeC1 || MODE == kModeGrad;
    static constexpr bool VDP = MODE == kModeGrad;
    static constexpr bool HASDP = SDP || VDP;
    static constexpr bool W2 = HASDP || MODE == kModeOut;        // second column-side tensor
    static constexpr bool ZW2 = MODE == kModeOut || MODE == kModeC1;  // vector operand = W2 tile
};

struct TcVecArgs {
    int H, L, h, D, BH;
    const int* jobs;            // job order (active row tiles first), or null for the natural order
    const uint32_t* tile_bits;  // [B][words]: 128-position tiles holding an active non-dustbin token
    int words;
    float sc2;              // scale * log2(e)
    const float* logm;
    const float* pr;        // natural row bias [BH, L]
    const float* pcm2;      // masked log2 column bias [BH, L]
    const float* pc;        // natural column bias (read at D)
    float* sout;
    const float* f;
    const float* hv;
    const float* m;
    void* vout;
    float vscale;
    const float* xr[kMaxMods];
    const float* yc[kMaxMods];
    const __nv_bfloat16* Zg;  // column-side vector operand (global), read at D
    const float* sd_term;
    const float* dp_term;
    uint32_t* status;
    // Row sweep only: the plan entries Pt of every band tile, bf16, in a tile-relative band store
    // (row r of row tile I at pcache[r * cpitch + (c - 128 I + h)], cpitch = 2 h + 128), or null.
    __nv_bfloat16* pcache;
    int cpitch;
    // Column sweep beta_R: partial row-side sums of Pt dP (see BwdPass::s1part), or null.
    float* s1part;
    size_t s1stride;
    int s1E;
};

constexpr int kSweepEpi = 16;         // epilogue warps: four per TMEM lane quadrant, 32 columns each
constexpr int kSweepThreads = 32 * (4 + kSweepEpi);   // TMA warp, S-MMA warp, epilogue warps, product-MMA warp, dP-MMA warp
constexpr int kSweepDpWarp = 3 + kSweepEpi;

template <int DH, int NV, bool FOLD = false>
struct SweepCfg {
    static constexpr int BM = 128, BN = 128;
    static constexpr int KATOMS = DH / 64;
    // Column tiles ride two rings.  The late ring holds the tile the product MMA reads (or, in
    // a pass without one, the dP operand) together with the column vectors the epilogue reads;
    // a slot comes back only after the product, so it gets three.  The early ring holds the
    // other tile, which is free as soon as its score MMA completes: one slot suffices.
    static constexpr int NL = 3, NE = 1;
    static constexpr uint32_t XB = BM * DH * 2;          // row tile bytes
    static constexpr uint32_t YB = BN * DH * 2;          // column tile bytes
    static constexpr uint32_t XATOM = BM * 128;          // one 64-element atom column of a row tile
    static constexpr uint32_t YATOM = BN * 128;          // ... of a column tile
    static constexpr uint32_t CB = BM * BN * 2;          // coefficient tile bytes (32 KB)
    static constexpr uint32_t CATOM = BM * 128;          // one 64-column atom of a coefficient tile
    static constexpr uint32_t VB = NV * BN * 4;          // column vector bytes per late-ring slot
    // The row tiles X and A land (TMA) in the coefficient buffers and are moved into TMEM
    // before the first coefficient is written.
    static constexpr uint32_t OFF_C = 0;
    static constexpr uint32_t OFF_L = 2 * CB;
    static constexpr uint32_t OFF_E = OFF_L + NL * YB;
    static constexpr uint32_t OFF_V = OFF_E + NE * YB;
    // Folded modifiers (dQ / dK): the row tile's and the early column tile's [128 x 16] bf16
    // modifier operands, 32-byte swizzled
    static constexpr uint32_t EXTB = 128 * 16 * 2;
    static constexpr uint32_t OFF_XE = (OFF_V + NL * VB + 1023) / 1024 * 1024;
    static constexpr uint32_t OFF_YE = OFF_XE + EXTB;
    static constexpr uint32_t OFF_RED = FOLD ? OFF_YE + EXTB : OFF_V + NL * VB;  // [2 sums][4 quarters][128 rows] scalar partials
    static constexpr uint32_t OFF_BAR = OFF_RED + 2 * 4 * 128 * 4;
    // full_l[NL] empty_l[NL] full_e empty_e xfull tfull tempty cfull[2] cempty[2] accfull xtm accempty jobdone
    static constexpr uint32_t NBARS = 2 * NL + 2 + 1 + 2 + 4 + 1 + 1 + 1 + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr uint32_t OFF_TILES = OFF_MISC + 64;
    static size_t smem_bytes(int max_tiles) { return 1024 + OFF_TILES + 2 * 4 * size_t(max_tiles); }
    static constexpr uint32_t IDESC_S = ptx::idesc_bf16(128, BN, false, false);
    static constexpr uint32_t IDESC_O = ptx::idesc_bf16(128, DH, false, true);
    // TMEM columns: the S and dP tiles (one buffer each: the epilogue reads a whole tile into
    // registers before any arithmetic and hands it back at once), the d-wide accumulator, and
    // the row tiles X and A as MMA A operands (one row per lane, two bf16 per column)
    static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_ACC = 256, TM_X = 384, TM_A = 448;
};

// FOLD (dQ / dK without a dustbin): the rank-2R modifier term sum_k xr_k yc_k^T comes out of the
// dP product itself, one more K = 16 step over [128 x 16] bf16 operand tiles XE (rows) and YE
// (columns) that carry each modifier split into hi + lo bf16 parts (see bwd_vectors_kernel), so
// the epilogue's coefficient is Pt * dP' with no per-entry modifier arithmetic.
template <int DH, int MODE, int NMOD, bool FOLD>
__global__ void __launch_bounds__(kSweepThreads, 1)
    tc_sweep_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmW,
                    const __grid_constant__ CUtensorMap tmXE, const __grid_constant__ CUtensorMap tmYE,
                    const TcVecArgs a, int max_tiles) {
    using M = ModeT<MODE>;
    static_assert(!FOLD || (MODE == kModeGrad && NMOD == 0), "folded modifiers are a dQ / dK form");
    constexpr int NV = 1 + (M::SM ? 1 : 0) + NMOD;   // column vectors per column tile: pcm2, m, yc...
    using C = SweepCfg<DH, NV, FOLD>;
    constexpr int VOFF_M = 1, VOFF_Y = 1 + (M::SM ? 1 : 0);
    // W rides the late ring when the product reads it or when there is no product (R2); Y when
    // the product reads Y (dQ / dK).
    constexpr bool LATE_W = !M::VEC || M::ZW2;
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = align1024(smraw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.L, h = a.h, D = a.D;
    (void)max_tiles;
    // Persistent: CTA c takes the jobs c, c + gridDim.x, ... (job = one 128-row tile of one unit,
    // BH L / 128 of them; neighbouring CTAs work on neighbouring row tiles at the same time, so
    // the column tiles they share are read from L2).  Every role walks the same jobs and, inside
    // a job, the same band tiles (those holding an active non-dustbin column, from the tile
    // bits), so ring slots and barrier phases follow from running counters across jobs; a job
    // whose row tile holds no active token only has its outputs zeroed.
    const int nT = L / C::BM, n_jobs = a.BH * nT;
    struct Job {
        int bh, b, r0, t_lo, t_hi;
        size_t base;
        const uint32_t* bits;
        bool act;
    };
    // Every role walks list positions blockIdx.x, blockIdx.x + gridDim.x, ...; the job at the next
    // position is read from the list one job ahead, so that its load is off the critical path.
    auto list_at = [&](int pos) { return (a.jobs && pos < n_jobs) ? __ldg(a.jobs + pos) : pos; };
    auto job_of = [&](int job) {
        Job j;
        j.bh = job / nT;
        j.b = j.bh / a.H;
        j.r0 = (job - j.bh * nT) * C::BM;
        j.base = size_t(j.bh) * L;
        j.bits = a.tile_bits + size_t(j.b) * a.words;
        j.act = tile_bit(j.bits, j.r0 / C::BM);
        j.t_lo = max(0, j.r0 - h) / C::BN;
        j.t_hi = min(L - 1, j.r0 + C::BM - 1 + h) / C::BN;
        return j;
    };

    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    const uint32_t bar0 = ptx::smem_u32(bars);
    auto full_l = [&](int s) { return bar0 + 8u * s; };
    auto empty_l = [&](int s) { return bar0 + 8u * (C::NL + s); };
    const uint32_t full_e = bar0 + 8u * (2 * C::NL);
    const uint32_t empty_e = bar0 + 8u * (2 * C::NL + 1);
    const uint32_t xfull = bar0 + 8u * (2 * C::NL + 2);
    const uint32_t tfull = bar0 + 8u * (2 * C::NL + 3);
    const uint32_t tempty = bar0 + 8u * (2 * C::NL + 4);
    auto cfull = [&](int i) { return bar0 + 8u * (2 * C::NL + 5 + i); };
    auto cempty = [&](int i) { return bar0 + 8u * (2 * C::NL + 7 + i); };
    const uint32_t accfull = bar0 + 8u * (2 * C::NL + 9);
    const uint32_t xtm = bar0 + 8u * (2 * C::NL + 10);       // row tiles copied into TMEM
    const uint32_t accempty = bar0 + 8u * (2 * C::NL + 11);  // accumulator read back
    // every score product of a job has completed (a pass without products: the next job's row
    // tiles may then overwrite TMEM).  One phase per job, committed after its last tile, so the
    // row-tile thread, which copies job k's tiles before phase k can start, is never more than
    // one phase behind it.  (Waiting instead on the per-tile barrier for each of the previous
    // job's tiles could block: once two of them had completed, the wait for the first had the
    // parity of the phase in progress and then waited for a tile of the next job, which needs
    // this very thread.)
    const uint32_t jobdone = bar0 + 8u * (2 * C::NL + 12);
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    if (tid == 0) {
        *abort_flag = 0;
        for (int s = 0; s < C::NL; ++s) {
            ptx::mbar_init(full_l(s), 1);
            // the epilogue warps (column vectors) + the product's commit, or in a pass without
            // one the dP issuer's
            ptx::mbar_init(empty_l(s), 1 + kSweepEpi);
        }
        ptx::mbar_init(full_e, 1);
        ptx::mbar_init(empty_e, 1);                 // the commit of the score MMA that reads it
        ptx::mbar_init(xfull, 1);
        ptx::mbar_init(tfull, M::HASDP ? 2 : 1);   // the S issuer and the dP issuer
        ptx::mbar_init(tempty, kSweepEpi);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(cfull(i), kSweepEpi);
            ptx::mbar_init(cempty(i), 1);
        }
        ptx::mbar_init(accfull, 1);
        ptx::mbar_init(xtm, 1);                     // the commit of the row tiles' copy into TMEM
        ptx::mbar_init(accempty, kSweepEpi / 2);   // the warps of column quarters 0 and 1
        ptx::mbar_init(jobdone, M::HASDP ? 2 : 1); // the S issuer and the dP issuer
        ptx::mbar_fence_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(misc), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tbase = misc[0];

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer: the column tiles of every job ----------------
            static_assert(M::W2, "every sweep pass reads two column-side tensors");
            ptx::prefetch_tmap(&tmY);
            ptx::prefetch_tmap(&tmW);
            if (FOLD) ptx::prefetch_tmap(&tmYE);
            const CUtensorMap* tm_late = LATE_W ? &tmW : &tmY;
            const CUtensorMap* tm_early = LATE_W ? &tmY : &tmW;
            const float* vsrc[NV];
            {
                int k = 0;
                vsrc[k++] = a.pcm2;
                if (M::SM) vsrc[k++] = a.m;
                for (int i = 0; i < NMOD; ++i) vsrc[k++] = a.yc[i];
            }
            constexpr uint32_t late_bytes = C::YB + uint32_t(NV) * C::BN * 4;
            int issued_l = 0, issued_e = 0, itg = 0;
            bool ok = true;
            int jnext = list_at(blockIdx.x);
            for (int job = blockIdx.x; job < n_jobs && ok; job += gridDim.x) {
                const int jcur = jnext;
                jnext = list_at(job + gridDim.x);
                const Job jb = job_of(jcur);
                if (!jb.act) continue;
                for (int t = jb.t_lo; t <= jb.t_hi; ++t) {
                    if (!tile_bit(jb.bits, t)) continue;
                    const int it = itg++;
                    const int sl = it % C::NL;
                    const int c0 = t * C::BN;
                    // late ring: column tile + column vectors
                    if (!ptx::mbar_wait(empty_l(sl), ((it / C::NL) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                    ptx::mbar_expect_tx(full_l(sl), late_bytes);
                    const uint32_t ls = ptx::smem_u32(sm + C::OFF_L + sl * C::YB);
                    for (int ka = 0; ka < C::KATOMS; ++ka)
                        ptx::tma_load_2d(ls + ka * C::YATOM, tm_late, ka * 64, int(jb.base) + c0, full_l(sl));
                    const uint32_t vs = ptx::smem_u32(sm + C::OFF_V + sl * C::VB);
#pragma unroll
                    for (int i = 0; i < NV; ++i)
                        ptx::bulk_load(vs + i * C::BN * 4, vsrc[i] + jb.base + c0, C::BN * 4, full_l(sl));
                    issued_l = it + 1;
                    // early ring: the other column tile
                    if (!ptx::mbar_wait(empty_e, (it & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                    ptx::mbar_expect_tx(full_e, C::YB + (FOLD ? C::EXTB : 0u));
                    const uint32_t es = ptx::smem_u32(sm + C::OFF_E);
                    for (int ka = 0; ka < C::KATOMS; ++ka)
                        ptx::tma_load_2d(es + ka * C::YATOM, tm_early, ka * 64, int(jb.base) + c0, full_e);
                    // (the dP operand rides the early ring in dQ / dK: its modifier tile goes with it)
                    if (FOLD) ptx::tma_load_2d(ptx::smem_u32(sm + C::OFF_YE), &tmYE, 0, int(jb.base) + c0, full_e);
                    issued_e = it + 1;
                }
            }
            if (*abort_flag) {
                // let every copy still in flight land before the CTA can exit
                volatile int dummy = 0;
                for (int it = max(0, issued_l - C::NL); it < issued_l; ++it)
                    ptx::mbar_wait(full_l(it % C::NL), (it / C::NL) & 1, &dummy, a.status);
                if (issued_e > 0) ptx::mbar_wait(full_e, (issued_e - 1) & 1, &dummy, a.status);
            }
        }
    } else if (warp == 1 || warp == kSweepDpWarp) {
        // ---------------- score MMA issuers: S (warp 1) and dP (warp kSweepDpWarp) tiles ----------------
        // One thread each, so that neither product waits behind the other's instruction stream.
        const bool is_dp = warp == kSweepDpWarp;
        if (lane == 0 && (!is_dp || M::HASDP)) {
            int issued = 0, itg = 0, jc = 0;
            bool ok = true;
            const uint32_t dtm = tbase + (is_dp ? C::TM_DP : C::TM_S);
            const uint32_t atm = tbase + (is_dp ? C::TM_A : C::TM_X);
            const bool late = is_dp == LATE_W;   // this issuer's column tile (W for dP, Y for S) rides the late ring
            int jnext = list_at(blockIdx.x);
            for (int job = blockIdx.x; job < n_jobs && ok; job += gridDim.x) {
                const int jcur = jnext;
                jnext = list_at(job + gridDim.x);
                const Job jb = job_of(jcur);
                if (!jb.act) continue;
                // this job's row tiles are in TMEM (copied once they had landed, with the row
                // modifier tile XE that the dP product reads from shared memory)
                ok = ptx::mbar_wait(xtm, jc & 1, abort_flag, a.status);
                ++jc;
                if (!ok) break;
                ptx::tc_fence_after();
                for (int t = jb.t_lo; t <= jb.t_hi && ok; ++t) {
                    if (!tile_bit(jb.bits, t)) continue;
                    const int it = itg++;
                    const int sl = it % C::NL;
                    const bool got = late ? ptx::mbar_wait(full_l(sl), (it / C::NL) & 1, abort_flag, a.status)
                                          : ptx::mbar_wait(full_e, it & 1, abort_flag, a.status);
                    if (!got) { ok = false; break; }
                    if (!ptx::mbar_wait(tempty, (it & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
                    ptx::tc_fence_after();
                    // B operand: the column tile of S (Y) or of dP (W); A operand (row tile) from TMEM,
                    // 8 columns per K step of 16
                    const uint32_t boff = late ? C::OFF_L + uint32_t(sl) * C::YB : C::OFF_E;
                    const uint64_t bd = ptx::smem_desc(ptx::smem_u32(sm + boff), 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk) {
                        const uint64_t bo = uint64_t(((kk >> 2) * C::YATOM + (kk & 3) * 32) >> 4);
                        ptx::mma_bf16_ts(dtm, atm + uint32_t(kk * 8), bd + bo, C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    // dP' = dP + XE YE^T = dP - sum_k xr_k yc_k^T
                    if (FOLD && is_dp)
                        ptx::mma_bf16(dtm, ptx::smem_desc_sw32(ptx::smem_u32(sm + C::OFF_XE)),
                                      ptx::smem_desc_sw32(ptx::smem_u32(sm + C::OFF_YE)), C::IDESC_S, 1u);
                    ptx::mma_commit(tfull);
                    // the early tile is free once this product completes; a late slot normally comes
                    // back after the product MMA, or here in a pass without one
                    if (!late) ptx::mma_commit(empty_e);
                    else if (!M::VEC) ptx::mma_commit(empty_l(sl));
                    issued = it + 1;
                }
                if (!M::VEC && ok) ptx::mma_commit(jobdone);
            }
            if (*abort_flag && issued > 0) {
                volatile int dummy = 0;
                ptx::mbar_wait(tfull, (issued - 1) & 1, &dummy, a.status);
            }
        }
    } else if (warp == 2 + kSweepEpi) {
        if (lane == 0) {
            // ---------------- row tiles into TMEM and the product MMA issuer ----------------
            // The row tiles X and A of a job land (TMA) in the coefficient buffers and are copied
            // from there into TMEM as MMA A operands (tcgen05.cp, one row per lane, two bf16 per
            // 32-bit column; committed to xtm).  The next job's copy starts once this job's
            // products are done (the coefficient buffers are free and every score product that
            // read the TMEM row tiles has completed), or, in a pass without products, once its
            // last score tile has completed, so the next job's scores overlap this job's
            // read-back.  The products acc += coef(j) * Z(j) have a thread of their own, so that
            // score tiles are never queued behind a product that waits for the epilogue
            // (tcgen05.commit tracks the issuing thread's MMAs).
            ptx::prefetch_tmap(&tmX);
            if (M::HASDP) ptx::prefetch_tmap(&tmA);
            if (FOLD) ptx::prefetch_tmap(&tmXE);
            int done = 0, itg = 0, jc = 0;
            bool ok = true, xpending = false;
            int jnext = list_at(blockIdx.x);
            for (int job = blockIdx.x; job < n_jobs && ok; job += gridDim.x) {
                const int jcur = jnext;
                jnext = list_at(job + gridDim.x);
                const Job jb = job_of(jcur);
                if (!jb.act) continue;
                if (jc > 0) {
                    // the previous job's products (or, in a pass without them, its score
                    // products) are done with the TMEM row tiles and the coefficient buffers
                    ok = ptx::mbar_wait(M::VEC ? accfull : jobdone, (jc - 1) & 1, abort_flag, a.status);
                    if (!ok) break;
                }
                const uint32_t xs = ptx::smem_u32(sm + C::OFF_C), as = xs + C::XB;
                ptx::mbar_expect_tx(xfull, C::XB * (M::HASDP ? 2 : 1) + (FOLD ? C::EXTB : 0u));
                for (int ka = 0; ka < C::KATOMS; ++ka) {
                    ptx::tma_load_2d(xs + ka * C::XATOM, &tmX, ka * 64, int(jb.base) + jb.r0, xfull);
                    if (M::HASDP) ptx::tma_load_2d(as + ka * C::XATOM, &tmA, ka * 64, int(jb.base) + jb.r0, xfull);
                }
                if (FOLD) ptx::tma_load_2d(ptx::smem_u32(sm + C::OFF_XE), &tmXE, 0, int(jb.base) + jb.r0, xfull);
                xpending = true;
                if (!ptx::mbar_wait(xfull, jc & 1, abort_flag, a.status)) { ok = false; break; }
                xpending = false;
                ptx::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < DH / 16; ++kk) {
                    const uint32_t koff = uint32_t((kk >> 2) * C::XATOM + (kk & 3) * 32);
                    ptx::tmem_cp_128x256b(tbase + C::TM_X + uint32_t(kk * 8), ptx::smem_desc(xs + koff, 16, 1024));
                    if (M::HASDP)
                        ptx::tmem_cp_128x256b(tbase + C::TM_A + uint32_t(kk * 8), ptx::smem_desc(as + koff, 16, 1024));
                }
                ptx::mma_commit(xtm);
                if (M::VEC) {
                    // the previous job's accumulator has been read back
                    if (jc > 0 && !ptx::mbar_wait(accempty, (jc - 1) & 1, abort_flag, a.status)) { ok = false; break; }
                    int j = 0;
                    for (int t = jb.t_lo; t <= jb.t_hi && ok; ++t) {
                        if (!tile_bit(jb.bits, t)) continue;
                        const int it = itg++;
                        const int cb = it & 1;
                        if (!ptx::mbar_wait(cfull(cb), (it >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
                        ptx::tc_fence_after();
                        const int sl = it % C::NL;
                        const uint32_t zs = ptx::smem_u32(sm + C::OFF_L + sl * C::YB);   // Z rides the late ring
                        const uint32_t cs = ptx::smem_u32(sm + C::OFF_C + cb * C::CB);
#pragma unroll
                        for (int kk = 0; kk < C::BN / 16; ++kk)
                            ptx::mma_bf16(tbase + C::TM_ACC, ptx::smem_desc(cs + (kk >> 2) * C::CATOM + (kk & 3) * 32, 16, 1024),
                                          ptx::smem_desc(zs + kk * 2048, C::YATOM, 1024), C::IDESC_O,
                                          (j > 0 || kk > 0) ? 1u : 0u);
                        ptx::mma_commit(cempty(cb));
                        ptx::mma_commit(empty_l(sl));
                        done = it + 1;
                        ++j;
                    }
                    if (ok) ptx::mma_commit(accfull);
                }
                ++jc;
            }
            if (*abort_flag) {
                volatile int dummy = 0;
                if (M::VEC && done > 0) ptx::mbar_wait(cempty((done - 1) & 1), ((done - 1) >> 1) & 1, &dummy, a.status);
                // no row-tile copy may still be writing this CTA's shared memory when it exits
                if (xpending) ptx::mbar_wait(xfull, jc & 1, &dummy, a.status);
            }
        }
    } else {
        // ---------------- epilogue: warps 2..17, four per TMEM lane quadrant ----------------
        const int q = warp & 3;                  // lane quadrant
        const int qt = (warp - 2) >> 2;          // which 32 columns of each 128-column tile
        const int half = qt;                     // (quarters 0, 1 also read back the accumulator halves)
        const int row = q * 32 + lane;
        const uint32_t lane_base = uint32_t(q * 32) << 16;
        const uint32_t crow = uint32_t(row >> 3) * 1024u + uint32_t(row & 7) * 128u;
        const int etid = tid - 64;               // 0 .. 511
        const uint64_t SC2 = ptx::f2(a.sc2, a.sc2);
        int itg = 0, jc = 0;
        bool ok = true;
        int jnext = list_at(blockIdx.x);
        for (int job = blockIdx.x; job < n_jobs; job += gridDim.x) {
        const int jcur = jnext;
        jnext = list_at(job + gridDim.x);
        const Job jb = job_of(jcur);
        const int r0 = jb.r0;
        const size_t base = jb.base;
        if (!jb.act) {
            // no active token in this row tile: zero outputs
            if (M::SCAL)
                for (int i = etid; i < C::BM; i += 32 * kSweepEpi) a.sout[base + r0 + i] = 0.f;
            if (M::VEC) {
                __nv_bfloat16* vo = static_cast<__nv_bfloat16*>(a.vout) + (base + r0) * DH;
                for (int e = etid; e < C::BM * DH / 8; e += 32 * kSweepEpi)
                    reinterpret_cast<uint4*>(vo)[e] = make_uint4(0, 0, 0, 0);
            }
            continue;
        }
        const float* logm = a.logm + size_t(jb.b) * L;
        const int r = r0 + row;
        const float lm = logm[r];
        const bool ract = lm != kNegInf;
        const bool is_dustbin_row = (r == D) && ract;
        const float pr2 = ract ? a.pr[base + r] * kLog2e : kNegInf;
        const uint64_t PR2 = ptx::f2(pr2, pr2);
        float xr[NMOD > 0 ? NMOD : 1];
#pragma unroll
        for (int k = 0; k < NMOD; ++k) xr[k] = ract ? -a.xr[k][base + r] : 0.f;
        uint64_t s1a[2] = {ptx::f2(0.f, 0.f), ptx::f2(0.f, 0.f)};
        uint64_t s2a[2] = {ptx::f2(0.f, 0.f), ptx::f2(0.f, 0.f)};
        // (the row tiles reach TMEM by tcgen05.cp from the coefficient buffers: the first score
        // tile of the job, which this warp waits for, completes after that copy has read them)
        // Every epilogue warp has finished the previous job, whose scalar partials the warps of
        // column quarter 0 read after the shared-memory exchange below, before any warp writes
        // this job's (a job of one tile would otherwise let a fast warp overwrite them).
        ptx::named_bar_sync(2, 32 * kSweepEpi);
        for (int tcol = jb.t_lo; tcol <= jb.t_hi; ++tcol) {
            if (!tile_bit(jb.bits, tcol)) continue;
            const int it = itg++;
            if (!ok) continue;
                const int sl = it % C::NL, cb = it & 1;
                const int c0 = tcol * C::BN;
                // This warp's 32 x 32 block (rows r0 + 32 q .., columns c0 + 32 qt ..) against the band:
                // 0 = outside for every entry (no TMEM read, no exponentials; zero coefficients),
                // 1 = inside for every entry, 2 = cut by the band edge (masked per entry).
                const int dmin = c0 + qt * 32 - (r0 + q * 32 + 31), dmax = c0 + qt * 32 + 31 - (r0 + q * 32);
                const int cls = (dmin > h || dmax < -h) ? 0 : (dmax <= h && dmin >= -h) ? 1 : 2;
                // Waits are made warp-uniform: the tcgen05.ld below is a warp-collective (.aligned).
                bool w1 = ptx::mbar_wait(full_l(sl), (it / C::NL) & 1, abort_flag, a.status);   // column vectors
                bool w2 = w1 && ptx::mbar_wait(tfull, it & 1, abort_flag, a.status);
                bool w3 = w2 && (!M::VEC || ptx::mbar_wait(cempty(cb), ((it >> 1) & 1) ^ 1, abort_flag, a.status));
                if (!__all_sync(0xffffffffu, w3)) { ok = false; break; }
                ptx::tc_fence_after();
                // column vectors of this tile's late-ring slot (explicit shared-memory loads: the aligned base
                // pointer no longer carries the address space)
                const uint32_t cva = ptx::smem_u32(sm + C::OFF_V + sl * C::VB);
                auto cvec = [&](int vec, int col) { return ptx::ld_shared_f4(cva + uint32_t((vec * C::BN + col) * 4)); };
                const uint32_t cbase = ptx::smem_u32(sm + C::OFF_C + cb * C::CB) + uint32_t(qt >> 1) * C::CATOM + crow;
                if (cls == 0) {
                    // nothing of this block is in the band: hand the scores back unread; the product
                    // reads zeros for it
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(tempty);
                    if (M::VEC) {
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const uint32_t unit = uint32_t((qt & 1) * 4 + t);
                            ptx::st_shared_v4(cbase + ((unit ^ uint32_t(row & 7)) << 4), 0u, 0u, 0u, 0u);
                        }
                    }
                } else {
                // this warp's 32 columns of S (and dP), read whole; the buffer goes back at once
                float v[1][32], w[1][32];
                const uint32_t tl = tbase + lane_base + uint32_t(qt * 32);
                ptx::tmem_ld32(tl + C::TM_S, v[0]);
                if (M::HASDP) ptx::tmem_ld32(tl + C::TM_DP, w[0]);
                ptx::tmem_wait_ld(v[0]);
                if (M::HASDP) ptx::tmem_tie(w[0]);
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(tempty);
#pragma unroll
                for (int ch = 0; ch < 1; ++ch) {
                    const int cc0 = qt * 32;
                    float (&vc)[32] = v[ch];
                    float (&wc)[32] = w[ch];
                    // P~ = exp2(S * scale * log2e + row bias + column bias), pairs in fp32x2
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4) {
                        const float4 b4 = cvec(0, cc0 + 4 * j4);
                        uint64_t x0 = ptx::ffma2(ptx::f2(vc[4 * j4 + 0], vc[4 * j4 + 1]), SC2, ptx::fadd2(PR2, ptx::f2(b4.x, b4.y)));
                        uint64_t x1 = ptx::ffma2(ptx::f2(vc[4 * j4 + 2], vc[4 * j4 + 3]), SC2, ptx::fadd2(PR2, ptx::f2(b4.z, b4.w)));
                        ptx::f2split(x0, vc[4 * j4 + 0], vc[4 * j4 + 1]);
                        ptx::f2split(x1, vc[4 * j4 + 2], vc[4 * j4 + 3]);
                    }
                    if (cls == 2) {
                        const int dlt0 = c0 + cc0 - r;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int dl = dlt0 + j;
                            if (dl < -h || dl > h) vc[j] = kNegInf;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) vc[j] = ptx::ex2(vc[j]);
                    if (MODE == kModeR2 && a.pcache) {
                        // cache this chunk of the plan: 32 entries of row r, 16-byte aligned (h % 8 == 0)
                        uint4* dst = reinterpret_cast<uint4*>(a.pcache + (base + r) * size_t(a.cpitch) + (c0 + cc0 - r0 + h));
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            dst[t] = make_uint4(ptx::pack_bf16(vc[8 * t], vc[8 * t + 1]), ptx::pack_bf16(vc[8 * t + 2], vc[8 * t + 3]),
                                                ptx::pack_bf16(vc[8 * t + 4], vc[8 * t + 5]), ptx::pack_bf16(vc[8 * t + 6], vc[8 * t + 7]));
                    }
                    if (M::SCAL) {
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const uint64_t P2 = ptx::f2(vc[2 * k], vc[2 * k + 1]);
                            if (M::SDP) s1a[k & 1] = ptx::ffma2(P2, ptx::f2(wc[2 * k], wc[2 * k + 1]), s1a[k & 1]);
                            if (M::SM) {
                                const float4 mv = cvec(VOFF_M, cc0 + 4 * (k >> 1));
                                s2a[k & 1] = ptx::ffma2(P2, (k & 1) ? ptx::f2(mv.z, mv.w) : ptx::f2(mv.x, mv.y), s2a[k & 1]);
                            }
                        }
                    }
                    if (M::VEC) {
                        // coefficient = P~ * (dP - sum_k xr_k yc_k)  (or P~ when the pass has no dP)
                        uint32_t pk[16];
#pragma unroll
                        for (int k4 = 0; k4 < 8; ++k4) {
                            uint64_t cf0 = M::VDP ? ptx::f2(wc[4 * k4], wc[4 * k4 + 1]) : ptx::f2(1.f, 1.f);
                            uint64_t cf1 = M::VDP ? ptx::f2(wc[4 * k4 + 2], wc[4 * k4 + 3]) : ptx::f2(1.f, 1.f);
#pragma unroll
                            for (int mm = 0; mm < NMOD; ++mm) {
                                const float4 yv = cvec(VOFF_Y + mm, cc0 + 4 * k4);
                                const uint64_t X2 = ptx::f2(xr[mm], xr[mm]);
                                cf0 = ptx::ffma2(X2, ptx::f2(yv.x, yv.y), cf0);
                                cf1 = ptx::ffma2(X2, ptx::f2(yv.z, yv.w), cf1);
                            }
                            float c0f, c1f, c2f, c3f;
                            ptx::f2split(cf0, c0f, c1f);
                            ptx::f2split(cf1, c2f, c3f);
                            pk[2 * k4] = ptx::pack_bf16(vc[4 * k4] * c0f, vc[4 * k4 + 1] * c1f);
                            pk[2 * k4 + 1] = ptx::pack_bf16(vc[4 * k4 + 2] * c2f, vc[4 * k4 + 3] * c3f);
                        }
                        // 128-byte-swizzled K-major tile: 16-byte unit u of a row at (u ^ (row & 7))
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const uint32_t unit = uint32_t((qt & 1) * 4 + t);
                            ptx::st_shared_v4(cbase + ((unit ^ uint32_t(row & 7)) << 4), pk[4 * t], pk[4 * t + 1],
                                              pk[4 * t + 2], pk[4 * t + 3]);
                        }
                    }
                    if (MODE == kModeC1 && a.s1part) {
                        // Pt dP summed over this warp's 32 rows for each of its 32 columns: a transposing
                        // butterfly (each step keeps half of the columns and adds the partner lane's copy
                        // of them), after which lane l holds column cc0 + l.  wc is free by now.
#pragma unroll
                        for (int j = 0; j < 32; ++j) wc[j] *= vc[j];
                        const int lb = lane;
#pragma unroll
                        for (int off = 16; off >= 1; off >>= 1) {
                            const bool up = (lb & off) != 0;
#pragma unroll
                            for (int i = 0; i < off; ++i) {
                                const float send = up ? wc[i] : wc[i + off];
                                const float keep = up ? wc[i + off] : wc[i];
                                wc[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                            }
                        }
                        const int slot = (tcol - jb.r0 / C::BM + a.s1E) * 4 + q;
                        a.s1part[size_t(slot) * a.s1stride + base + size_t(c0 + cc0 + lane)] = wc[0];
                    }
                }
                }   // cls != 0
                if (M::VEC) ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(empty_l(sl));
                    if (M::VEC) ptx::mbar_arrive(cfull(cb));
                }
        }
            // Scalar partials of the four column quarters meet in shared memory.
            float* red = reinterpret_cast<float*>(sm + C::OFF_RED);
            if (M::SCAL) {
                float a0, a1, b0, b1;
                ptx::f2split(ptx::fadd2(s1a[0], s1a[1]), a0, a1);
                ptx::f2split(ptx::fadd2(s2a[0], s2a[1]), b0, b1);
                red[(0 * 4 + qt) * 128 + row] = a0 + a1;
                red[(1 * 4 + qt) * 128 + row] = b0 + b1;
            }
            ptx::named_bar_sync(1, 32 * kSweepEpi);
            ok = __all_sync(0xffffffffu, ok);
            // Dustbin link of this row (the dustbin column), then the writes.
            const bool d_act = D >= 0 && logm[D] != kNegInf;
            float Pd = 0.f, dpd = 0.f, coefd = 0.f;
            if (ract && d_act && !is_dustbin_row) {
                Pd = ptx::ex2((a.sd_term[base + r] + a.pr[base + r] + a.pc[base + D]) * kLog2e);
                if (M::HASDP) dpd = a.dp_term[base + r];
                float mod = M::VDP ? dpd : 1.f;
#pragma unroll
                for (int k = 0; k < NMOD; ++k) mod += xr[k] * a.yc[k][base + D];
                coefd = Pd * mod;
            }
            if (M::SCAL && ok && qt == 0 && !is_dustbin_row) {
                float s1 = (red[0 * 128 + row] + red[1 * 128 + row]) + (red[2 * 128 + row] + red[3 * 128 + row]);
                float s2 = (red[4 * 128 + row] + red[5 * 128 + row]) + (red[6 * 128 + row] + red[7 * 128 + row]);
                if (d_act && ract) {
                    if (M::SDP) s1 = fmaf(Pd, dpd, s1);
                    if (M::SM) s2 = fmaf(Pd, a.m[base + D], s2);
                }
                float outv = 0.f;
                if (ract) {
                    outv = (a.f ? a.f[base + r] : 1.f) * (s1 + (a.hv ? a.hv[base + r] : 0.f) * s2);
                    if (!isfinite(outv)) atomicOr(a.status, kStatusNonFinite);
                }
                a.sout[base + r] = outv;
            }
            // The accumulator read is a warp-collective: every lane takes part; only the stores
            // are predicated (the dustbin row is written by the dense dustbin kernel).
            if (M::VEC && ok && qt < 2) {
                const bool have_acc = true;   // an active row tile holds its own diagonal tile
                bool wacc = ptx::mbar_wait(accfull, jc & 1, abort_flag, a.status);
                ok = __all_sync(0xffffffffu, wacc);
                ptx::tc_fence_after();
                if (ok) {
                    __nv_bfloat16* vo = static_cast<__nv_bfloat16*>(a.vout) + (base + r) * DH;
                    const __nv_bfloat16* zD = d_act ? a.Zg + (base + D) * DH : nullptr;
                    const bool store = !is_dustbin_row;
#pragma unroll
                    for (int chh = 0; chh < DH / 64; ++chh) {
                        const int col = half * (DH / 2) + chh * 32;
                        float v[32];
                        if (have_acc) {
                            ptx::tmem_ld32(tbase + lane_base + C::TM_ACC + uint32_t(col), v);
                            ptx::tmem_wait_ld(v);
                            if (chh == DH / 64 - 1) {
                                // the accumulator is read: the next job's products may start
                                ptx::tc_fence_before();
                                __syncwarp();
                                if (lane == 0) ptx::mbar_arrive(accempty);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = 0.f;
                        }
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            float lo = v[2 * j], hi = v[2 * j + 1];
                            if (ract && d_act && store) {
                                lo = fmaf(coefd, __bfloat162float(zD[col + 2 * j]), lo);
                                hi = fmaf(coefd, __bfloat162float(zD[col + 2 * j + 1]), hi);
                            }
                            pk[j] = ract ? ptx::pack_bf16(a.vscale * lo, a.vscale * hi) : 0u;
                        }
                        if (store) {
                            uint4* dst = reinterpret_cast<uint4*>(vo + col);
#pragma unroll
                            for (int t = 0; t < 4; ++t)
                                dst[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
                        }
                    }
                }
            }
        ++jc;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tbase, 512);
    }
}

int max_tiles_for(int L, int h, int BM, int BN) {
    const long span = long(BM) + 2L * h;
    const long t = span / BN + 2;
    return int(std::min<long>(t, L / BN));
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
}

}  // namespace

// The sweep kernel keeps its band's tile list in shared memory: very wide bands (W beyond
// about 7e4, with L longer than that) do not fit next to the tiles and run on the CUDA-core
// kernels instead.
constexpr size_t kMaxSmem = 227 * 1024;
bool tc_supported(const Geom& g) {
    if (g.dtype != EOT_BF16 || (g.d != 64 && g.d != 128) || encode_fn() == nullptr) return false;
    const int mt = max_tiles_for(g.L, g.h, 128, 128);
    return SweepCfg<128, 1 + kMaxMods>::smem_bytes(mt) <= kMaxSmem;
}

bool tma_map_bf16(CUtensorMap* m, const void* base, uint64_t rows, int d, int box_rows) {
    return make_map(m, base, rows, d, box_rows);
}

int sm_count() {
    static int n = [] {
        int dev = 0, v = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        return v;
    }();
    return n;
}

template <int DH, int KIND, bool MULTI, bool EXT = false>
cudaError_t launch_band_variant(const CUtensorMap& tmX, const CUtensorMap& tmY, const CUtensorMap& tmUE,
                                const CUtensorMap& tmVE, const TcBandArgs& a, int grid, cudaStream_t st) {
    constexpr size_t smem = BandCfg<DH, KIND, EXT>::SMEM;
    auto kernel = tc_band_kernel<DH, KIND, MULTI, EXT>;
    cudaError_t e = set_smem(kernel, smem);
    if (e != cudaSuccess) return e;
    // the register split inside the kernel assumes this launch allocation
    cudaFuncAttributes fa{};
    if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return e;
    if (fa.numRegs != kBandLaunchRegs) return cudaErrorNotSupported;
    if (!MULTI) {
        kernel<<<grid, kBandThreads, smem, st>>>(tmX, tmY, tmUE, tmVE, a);
        return cudaGetLastError();
    }
    // fused half-steps meet at grid-wide barriers: every CTA must be resident at once
    void* args[] = {const_cast<CUtensorMap*>(&tmX), const_cast<CUtensorMap*>(&tmY), const_cast<CUtensorMap*>(&tmUE),
                    const_cast<CUtensorMap*>(&tmVE), const_cast<TcBandArgs*>(&a)};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3(grid), dim3(kBandThreads), args,
                                       smem, st);
}

// Item ranges of the CTAs of a fused launch: contiguous, each holding about the same weight (from
// an item's active 128-row tiles, see weight below), so that units with few active tokens (padded sequences)
// do not leave some CTAs with all-active items and others with none.  bounds[c] = the first item
// i with (weight before i) * grid >= c * total; the last range runs to the end, so that every
// item (inactive ones write their rows) belongs to exactly one CTA.  One CTA of 1024 threads.
__device__ void band_bounds_block(const uint32_t* bits, int words, int H, int nT, int ppu, int n_items, int grid,
                                  int* bounds) {
    __shared__ int wsum[32];
    __shared__ int carry;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    auto weight = [&](int i) {
        const int bh = i / ppu, b = bh / H, p = i - bh * ppu;
        const uint32_t* bb = bits + size_t(b) * words;
        const int halves = int(tile_bit(bb, 2 * p)) + ((2 * p + 1 < nT) ? int(tile_bit(bb, 2 * p + 1)) : 0);
        // cost model, measured on a padded batch: an item's shared cost (its column tiles, waits
        // and decode) weighs like one of its active row halves, an inactive item (its rows
        // written as zeros) like a quarter of one
        return halves ? 4 + 4 * halves : 1;
    };
    // total weight
    int t = 0;
    for (int i = tid; i < n_items; i += blockDim.x) t += weight(i);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (lane == 0) wsum[wid] = t;
    for (int c = tid; c <= grid; c += blockDim.x) bounds[c] = 0;
    __syncthreads();
    long long total = 0;
    for (int k = 0; k < int(blockDim.x >> 5); ++k) total += wsum[k];
    if (tid == 0) carry = 0;
    __syncthreads();
    // inclusive scan of the weights in chunks of blockDim.x; item i owns the boundaries c with
    // E_i grid < c total <= (E_i + w_i) grid (E_i = weight before i): bounds[c] = i + 1
    for (int base = 0; base < n_items && total > 0; base += blockDim.x) {
        const int i = base + tid;
        const int w = i < n_items ? weight(i) : 0;
        int x = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        __syncthreads();                       // wsum of the previous chunk is read
        if (lane == 31) wsum[wid] = x;
        __syncthreads();
        int before = carry;
        for (int k = 0; k < wid; ++k) before += wsum[k];
        const long long incl = before + x, excl = incl - w;
        if (w > 0) {
            const long long c_lo = excl * grid / total + 1;
            const long long c_hi = incl * grid / total < grid ? incl * grid / total : (long long)grid;
            for (long long c = c_lo; c <= c_hi; ++c) bounds[c] = i + 1;
        }
        __syncthreads();
        if (tid == blockDim.x - 1) carry = int(incl);
        __syncthreads();
    }
    __syncthreads();
    if (tid == 0) {
        bounds[0] = 0;
        bounds[grid] = n_items;
    }
}

// CTAs of a band launch: one per SM, at most one per item.
int band_grid(const Geom& g) {
    const int n_items = g.BH * ((g.L / 128 + 1) / 2);
    return std::max(1, std::min({n_items, sm_count(), kMaxBandCtas}));
}

// Band row reduction over S = scale X Y^T (geometry, tile bits and the per-kind vectors in a);
// multi: the fused shifted half-steps a.hs0 .. a.hs0 + a.nhs - 1 in one cooperative launch.
cudaError_t launch_band(const Geom& g, const void* X, const void* Y, TcBandArgs a, int kind, cudaStream_t st,
                        bool multi = false) {
    if (!a.tile_bits) return cudaErrorInvalidValue;
    CUtensorMap tmX, tmY;
    const uint64_t rows = uint64_t(g.BH) * g.L;
    if (!make_map(&tmX, X, rows, g.d, 128) || !make_map(&tmY, Y, rows, g.d, 128)) return cudaErrorInvalidValue;
    // fused d = 128 half-steps read the column-bias operand rows of both sides
    CUtensorMap tmUE = tmX, tmVE = tmX;
    const bool ext = multi && g.d == 128 && g.h >= 256 && a.ue && a.ve;
    // a weighted band sum of a wide d = 128 band with its column bias as operand rows (in ue)
    const bool wext = !multi && kind == kBandWsum && g.d == 128 && g.h >= 256 && a.ue;
    if (ext) {
        if (!make_map_ext(&tmUE, a.ue, rows, 128) || !make_map_ext(&tmVE, a.ve, rows, 128)) return cudaErrorInvalidValue;
    } else if (wext) {
        if (!make_map_ext(&tmUE, a.ue, rows, 128)) return cudaErrorInvalidValue;
    } else if (multi) {
        a.ue = a.ve = nullptr;   // (no operand rows written either)
    }
    a.H = g.H;
    a.L = g.L;
    a.h = g.h;
    a.D = g.D;
    a.dself = g.dself;
    a.sl2 = g.scale * kLog2e;
    a.isl2 = float(1.0 / double(a.sl2));
    a.words = tile_words(g.L);
    a.pairs_per_unit = (g.L / 128 + 1) / 2;
    a.n_items = g.BH * a.pairs_per_unit;
    const int grid = band_grid(g);
    a.items_per_cta = (a.n_items + grid - 1) / grid;
    // (ranges of equal weight cover every CTA of the grid; equal ranges may leave the last empty)
    const int grid_used = a.bounds ? grid : (a.n_items + a.items_per_cta - 1) / a.items_per_cta;
    if (!multi) {
        a.hs0 = 0;
        a.nhs = 1;
    } else if (kind != kBandShift || !a.gbar || a.nhs < 1 ||
               (g.D >= 0 && (!a.sd_row || !a.sd_col || !a.dpart || !a.dcnt ||
                             2 * size_t(a.pairs_per_unit) > size_t(dustbin_splits(g.L)) * size_t(g.d + 2)))) {
        return cudaErrorInvalidValue;
    }
    if (g.d == 128) {
        if (multi)
            return ext ? launch_band_variant<128, kBandShift, true, true>(tmX, tmY, tmUE, tmVE, a, grid_used, st)
                       : launch_band_variant<128, kBandShift, true, false>(tmX, tmY, tmUE, tmVE, a, grid_used, st);
        switch (kind) {
            case kBandOnline: return launch_band_variant<128, kBandOnline, false>(tmX, tmY, tmUE, tmVE, a, grid_used, st);
            case kBandShift: return launch_band_variant<128, kBandShift, false>(tmX, tmY, tmUE, tmVE, a, grid_used, st);
            case kBandWsum:
                return wext ? launch_band_variant<128, kBandWsum, false, true>(tmX, tmY, tmUE, tmVE, a, grid_used, st)
                            : launch_band_variant<128, kBandWsum, false>(tmX, tmY, tmUE, tmVE, a, grid_used, st);
        }
    } else {
        if (multi) return launch_band_variant<64, kBandShift, true>(tmX, tmY, tmUE, tmVE, a, grid_used, st);
        switch (kind) {
            case kBandOnline: return launch_band_variant<64, kBandOnline, false>(tmX, tmY, tmUE, tmVE, a, grid_used, st);
            case kBandShift: return launch_band_variant<64, kBandShift, false>(tmX, tmY, tmUE, tmVE, a, grid_used, st);
            case kBandWsum: return launch_band_variant<64, kBandWsum, false>(tmX, tmY, tmUE, tmVE, a, grid_used, st);
        }
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_tc_lse(const LsePass& p, cudaStream_t st) {
    TcBandArgs a{};
    a.logm = p.logm;
    a.tile_bits = p.tile_bits;
    a.colbias2 = p.colbias2;
    a.colpot = p.colpot;
    a.stab = p.stab;
    a.out = p.out;
    a.out_bias2 = p.out_bias2;
    a.pstride = p.pstride;
    a.sd_term = p.sd_term;
    a.status = p.status;
    a.ext_out = p.ext_out;
    a.bounds = p.bounds;
    cudaError_t e = launch_band(p.g, p.X, p.Y, a, p.stab ? kBandShift : kBandOnline, st);
    if (e != cudaSuccess || p.g.D < 0) return e;
    return launch_dustbin_lse(p, st);
}

cudaError_t launch_tc_lse_fused(const LsePass& row, const FusedSteps& f, cudaStream_t st) {
    if (!row.tile_bits) return cudaErrorInvalidValue;
    TcBandArgs a{};
    a.logm = row.logm;
    a.tile_bits = row.tile_bits;
    a.pstride = row.pstride;
    a.status = row.status;
    a.hs0 = f.hs0;
    a.nhs = f.nhs;
    a.T = f.T;
    a.u_tail = f.u_tail;
    a.v_tail = f.v_tail;
    a.ub2 = f.ub2;
    a.vb2 = f.vb2;
    a.gbar = f.gbar;
    a.sd_row = row.sd_term;
    a.sd_col = row.sd_dense;
    a.dpart = row.dpart;
    a.dcnt = row.dcnt;
    a.ue = f.ue;
    a.ve = f.ve;
    a.bounds = f.bounds;
    // row half-steps: X = Q (row.X), Y = K (row.Y); the kernel swaps them for column half-steps
    return launch_band(row.g, row.X, row.Y, a, kBandShift, st, true);
}

// Job order of the sweep kernel: the CTAs take jobs c, c + grid, ... of this list, so with the
// active row tiles first every CTA gets as many of them as any other (+-1) and neighbouring
// CTAs still work on neighbouring active tiles at the same time.  One CTA of 1024 threads:
// position of job i = (active jobs before i) if active, else (all active) + (inactive before i).
__device__ void sweep_jobs_block(const uint32_t* bits, int words, int H, int nT, int n_jobs, int* jobs) {
    __shared__ int wsum[32];
    __shared__ int carry;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    auto active = [&](int i) {
        const int bh = i / nT;
        return int(tile_bit(bits + size_t(bh / H) * words, i - bh * nT));
    };
    int t = 0;
    for (int i = tid; i < n_jobs; i += blockDim.x) t += active(i);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (lane == 0) wsum[wid] = t;
    __syncthreads();
    int n_act = 0;
    for (int k = 0; k < int(blockDim.x >> 5); ++k) n_act += wsum[k];
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < n_jobs; base += blockDim.x) {
        const int i = base + tid;
        const int a = i < n_jobs ? active(i) : 0;
        int x = a;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        __syncthreads();
        if (lane == 31) wsum[wid] = x;
        __syncthreads();
        int before = carry;
        for (int k = 0; k < wid; ++k) before += wsum[k];
        const int excl = before + x - a;           // active jobs before i
        if (i < n_jobs) jobs[a ? excl : n_act + (i - excl)] = i;
        __syncthreads();
        if (tid == blockDim.x - 1) carry = before + x;
        __syncthreads();
    }
}

// The band kernel's item ranges (CTA 0) and the sweep kernel's job order (CTA 1) of one problem,
// in one launch.
__global__ void __launch_bounds__(1024) schedule_kernel(const uint32_t* bits, int words, int H, int nT, int ppu,
                                                        int n_items, int grid, int* bounds, int n_jobs, int* jobs) {
    if (blockIdx.x == 0) band_bounds_block(bits, words, H, nT, ppu, n_items, grid, bounds);
    else sweep_jobs_block(bits, words, H, nT, n_jobs, jobs);
}

cudaError_t launch_schedule(const Geom& g, const uint32_t* tile_bits, int* bounds, int* jobs, cudaStream_t st) {
    if (!tile_bits || !bounds || !jobs) return cudaErrorInvalidValue;
    const int ppu = (g.L / 128 + 1) / 2, nT = g.L / 128;
    schedule_kernel<<<2, 1024, 0, st>>>(tile_bits, tile_words(g.L), g.H, nT, ppu, g.BH * ppu, band_grid(g), bounds,
                                        g.BH * nT, jobs);
    return cudaGetLastError();
}

struct ExtMaps {
    CUtensorMap xe, ye;
};

template <int DH, int MODE, int NMOD, bool FOLD = false>
cudaError_t launch_sweep(const CUtensorMap& tmX, const CUtensorMap& tmA, const CUtensorMap& tmY, const CUtensorMap& tmW,
                         const ExtMaps& ext, const TcVecArgs& a, int mt, dim3 grid, cudaStream_t st) {
    constexpr int NV = 1 + (ModeT<MODE>::SM ? 1 : 0) + NMOD;
    const size_t smem = SweepCfg<DH, NV, FOLD>::smem_bytes(mt);
    cudaError_t e = set_smem(tc_sweep_kernel<DH, MODE, NMOD, FOLD>, smem);
    if (e != cudaSuccess) return e;
    tc_sweep_kernel<DH, MODE, NMOD, FOLD><<<grid, kSweepThreads, smem, st>>>(tmX, tmA, tmY, tmW, ext.xe, ext.ye, a, mt);
    return cudaGetLastError();
}

template <int DH>
cudaError_t launch_sweep_dh(int mode, int nmod, bool fold, const CUtensorMap& tmX, const CUtensorMap& tmA,
                            const CUtensorMap& tmY, const CUtensorMap& tmW, const ExtMaps& ext, const TcVecArgs& a,
                            int mt, dim3 grid, cudaStream_t st) {
    if (fold) return mode == kModeGrad ? launch_sweep<DH, kModeGrad, 0, true>(tmX, tmA, tmY, tmW, ext, a, mt, grid, st)
                                       : cudaErrorInvalidValue;
    switch (mode) {
        case kModeOut: return launch_sweep<DH, kModeOut, 0>(tmX, tmA, tmY, tmW, ext, a, mt, grid, st);
        case kModeC1: return launch_sweep<DH, kModeC1, 0>(tmX, tmA, tmY, tmW, ext, a, mt, grid, st);
        case kModeR2: return launch_sweep<DH, kModeR2, 0>(tmX, tmA, tmY, tmW, ext, a, mt, grid, st);
        case kModeGrad:
            switch (nmod) {
                case 0: return launch_sweep<DH, kModeGrad, 0>(tmX, tmA, tmY, tmW, ext, a, mt, grid, st);
                case 2: return launch_sweep<DH, kModeGrad, 2>(tmX, tmA, tmY, tmW, ext, a, mt, grid, st);
                case 4: return launch_sweep<DH, kModeGrad, 4>(tmX, tmA, tmY, tmW, ext, a, mt, grid, st);
                case 8: return launch_sweep<DH, kModeGrad, 8>(tmX, tmA, tmY, tmW, ext, a, mt, grid, st);
                case 16: return launch_sweep<DH, kModeGrad, 16>(tmX, tmA, tmY, tmW, ext, a, mt, grid, st);
            }
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_tc_bwd(const BwdPass& p, cudaStream_t st) {
    const Geom& g = p.g;
    // Which pass this is (the orchestration in api.cu only builds these five kinds).
    int mode;
    if (p.vout && !p.sout && !p.v_dp && p.nmod == 0 && p.Z != p.Y) mode = kModeOut;
    else if (p.vout && p.sout && p.s_dp && !p.v_dp && p.nmod == 0 && p.Z == p.Bm) mode = kModeC1;
    else if (!p.vout && p.sout && p.s_dp && p.m) mode = kModeR2;
    else if (!p.vout && p.sout && !p.s_dp && p.m) mode = kModeStair;
    else if (p.vout && !p.sout && p.v_dp && p.Z == p.Y) mode = kModeGrad;
    else return cudaErrorInvalidValue;
    if (mode == kModeStair) {
        // f_r hv_r sum_c Pt_rc m_c: a weighted band row sum with row shift pr and column bias pc
        TcBandArgs a{};
        a.logm = p.logm;
        a.tile_bits = p.tile_bits;
        a.colbias2 = p.pcm2;
        a.colw = p.m;
        a.colpot = p.pc;
        a.stab = p.pr;
        a.out = p.sout;
        a.f = p.f;
        a.hv = p.hv;
        a.pstride = size_t(g.L);
        a.sd_term = p.sd_term;
        a.status = p.status;
        a.sadd = p.sadd;
        a.bounds = p.bounds;
        a.ue = const_cast<__nv_bfloat16*>(p.cext);   // read only (the column-bias operand rows)
        cudaError_t e = launch_band(g, p.X, p.Y, a, kBandWsum, st);
        if (e != cudaSuccess || g.D < 0) return e;
        return launch_dustbin_bwd(p, st);
    }
    // dQ / dK without a dustbin, with the modifiers prepared as hi / lo bf16 operand rows: fold
    // them into the dP product.
    const bool fold = mode == kModeGrad && p.xext && p.yext && g.D < 0 && p.nmod <= kMaxFoldMods;
    ExtMaps ext;
    // Modifier count rounded up to an instantiated one; the padding terms have xr = 0.
    int nmod = fold ? 0 : p.nmod;
    const int nmod_k = nmod == 0 ? 0 : nmod <= 2 ? 2 : nmod <= 4 ? 4 : nmod <= 8 ? 8 : 16;
    if (nmod_k > nmod && !p.zero_vec) return cudaErrorInvalidValue;
    const bool has_dp = mode == kModeC1 || mode == kModeR2 || mode == kModeGrad;
    const void* w2 = has_dp ? p.Bm : (mode == kModeOut ? p.Z : nullptr);
    const uint64_t rows = uint64_t(g.BH) * g.L;
    CUtensorMap tmX, tmA, tmY, tmW;
    if (!make_map(&tmX, p.X, rows, g.d, 128) || !make_map(&tmY, p.Y, rows, g.d, 128)) return cudaErrorInvalidValue;
    if (!make_map(&tmA, has_dp ? p.A : p.X, rows, g.d, 128)) return cudaErrorInvalidValue;
    if (!make_map(&tmW, w2 ? w2 : p.Y, rows, g.d, 128)) return cudaErrorInvalidValue;
    if (fold) {
        if (!make_map_ext(&ext.xe, p.xext, rows, 128) || !make_map_ext(&ext.ye, p.yext, rows, 128))
            return cudaErrorInvalidValue;
    } else {
        ext.xe = tmX;   // not read
        ext.ye = tmX;
    }
    TcVecArgs a{};
    a.H = g.H;
    a.L = g.L;
    a.h = g.h;
    a.D = g.D;
    a.sc2 = g.scale * kLog2e;
    a.logm = p.logm;
    a.pr = p.pr;
    a.pcm2 = p.pcm2;
    a.pc = p.pc;
    a.sout = p.sout;
    a.f = p.f;
    a.hv = p.hv;
    a.m = p.m;
    a.vout = p.vout;
    a.vscale = p.vscale;
    for (int k = 0; k < nmod_k; ++k) {
        a.xr[k] = k < nmod ? p.xr[k] : p.zero_vec;
        a.yc[k] = k < nmod ? p.yc[k] : p.zero_vec;
    }
    a.Zg = static_cast<const __nv_bfloat16*>(p.Z);
    a.sd_term = p.sd_term;
    a.dp_term = p.dp_term;
    a.status = p.status;
    a.pcache = mode == kModeR2 ? p.pcache : nullptr;
    a.cpitch = 2 * g.h + 128;
    a.s1part = mode == kModeC1 ? p.s1part : nullptr;
    a.s1stride = p.s1stride;
    a.s1E = p.s1E;
    if (!p.tile_bits) return cudaErrorInvalidValue;
    a.BH = g.BH;
    a.jobs = p.jobs;
    a.tile_bits = p.tile_bits;
    a.words = tile_words(g.L);
    const int mt = max_tiles_for(g.L, g.h, 128, 128);
    // persistent: one CTA per SM (or per job when there are fewer)
    const long n_jobs = long(g.BH) * (g.L / 128);
    dim3 grid(unsigned(std::max(1L, std::min<long>(n_jobs, sm_count()))));
    cudaError_t e = g.d == 128 ? launch_sweep_dh<128>(mode, nmod_k, fold, tmX, tmA, tmY, tmW, ext, a, mt, grid, st)
                               : launch_sweep_dh<64>(mode, nmod_k, fold, tmX, tmA, tmY, tmW, ext, a, mt, grid, st);
    if (e != cudaSuccess || g.D < 0) return e;
    return launch_dustbin_bwd(p, st);
}

}  // namespace eot
