// gqa_dec_kernel.cuh -- sm_100a GQA forward for few packed query rows (decode):
// at most 16 packed rows R = G*Tq per (batch, KV head), head dim 128.
//
// With so few query rows a 128-row MMA tile would be almost all padding, and so
// would the softmax work of one thread per query row.  Here both contractions are
// computed transposed ("swap AB"), so the 128 keys of a tile are the MMA's M
// dimension and the query rows its N = 16:
//
//   S' = K Q^T   [128 keys x 16 rows]   TMEM lanes = keys
//   O' = V^T P'  [128 dims x 16 rows]   TMEM lanes = head dims
//
// One softmax thread per key holds at most 16 scores of a tile; the row maxima
// are reduced over the 128 keys once per tile (warp butterfly, then the four
// warps through shared memory); each thread keeps partial row sums of its own
// keys, reduced once per segment.  P'^T (bf16, 16 rows x 128 keys, K-major,
// 128-byte swizzle) goes to shared memory as the B operand of the second MMA;
// V's shared-memory tile serves as the MN-major A operand V^T unchanged.
//
//   TMEM columns  [0,16) S'0   [16,32) S'1   [32,48) O'0   [48,64) O'1
//
// MMA order (one thread): S'(g), PV'(g-1), S'(g+1), PV'(g), ...  S' is double
// buffered; P' is double buffered; the softmax of tile g overlaps PV'(g-1).  O'
// is double buffered by segment (segment s accumulates in O'(s % 2)), so that the
// softmax goes on with the next segment while segment s is finished: its row
// statistics go to shared memory, and an epilogue warpgroup (warps 8-11, warp
// 8+q reading TMEM lane quadrant q) writes the output rows or the split piece,
// takes the piece's ticket and merges the row-block if the piece completes it.
// Warps: 0 Q/K producer (and the stream-K plan), 1 V producer, 2 TMEM owner +
// MMA issuer, 3 span-bounds table, 4-7 softmax (warp 4+q reads TMEM lane
// quadrant q), 8-11 epilogue.  The stream-K work split, the split partial slots
// and the last-arriver merge are those of the two-lane kernel (gqa_fwd2_kernel.cuh).
//
// FP8 K/V (FP8 = true; the AstrAI commit log's fp8 family stores tensors as E4M3
// with one scale per tensor): each K/V tile arrives by TMA as 128 keys x 128
// bytes in the upper half of its 32 KB stage, and four converter warps (8-11)
// widen it in place to the f16 layout the MMAs read (E4M3 -> f16 is exact),
// zeroing V rows past the logical length as they go; Q is converted from bf16
// to f16 in place once per segment, and P' is written as f16, so both MMAs run
// with f16 operands.  k_scale is folded into the logit scale and v_scale into
// the output normalisation.  With the converter warps in warps 8-11, the softmax
// warps run each segment's epilogue themselves (the same code, same barriers).
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "gqa_fwd2_kernel.cuh"

namespace gqa {

constexpr int NSOFT_DEC = 128;
constexpr int DEC_NQ = 16;  // N of both MMAs: packed query rows held (padded)

template <int NR_, bool PAGED_ = false, bool FP8_ = false>
struct DecCfg {
    static constexpr int D = 128, BN = 128, STK = 3, STV = 3, QBUF = 2;
    static constexpr int NR = NR_;  // query rows the softmax reads (8 or 16)
    static_assert(NR == 8 || NR == 16, "rows");
    static constexpr bool PAGED = PAGED_;
    static constexpr bool FP8 = FP8_;  // K/V stored as E4M3 bytes (contiguous caches only)
    static_assert(!(PAGED && FP8), "fp8 K/V over a paged cache is not built");
    static constexpr int NTHREADS = 384;  // + four epilogue warps (bf16) or converter warps (FP8)
    static constexpr bool EPIW = !FP8;    // a separate epilogue warpgroup runs the segment epilogues
    static constexpr int NBOX = D / 64;
    static constexpr int KV_BOX = BN * 128;             // one 64-column box of a K/V tile
    static constexpr int KV_BYTES = NBOX * KV_BOX;
    static constexpr int Q_BOX = DEC_NQ * 128;          // one 64-column box of the 16-row Q tile
    static constexpr int Q_BYTES = NBOX * Q_BOX;
    static constexpr int P_BOX = DEC_NQ * 128;          // one 64-key box of P'^T
    static constexpr int P_BYTES = (BN / 64) * P_BOX;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + STK * KV_BYTES;
    static constexpr int OFF_Q = OFF_V + STV * KV_BYTES;
    static constexpr int OFF_P = OFF_Q + QBUF * Q_BYTES;
    static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
    static constexpr int B_QFULL = 0;                   // [QBUF]
    static constexpr int B_QEMPTY = B_QFULL + QBUF;     // [QBUF]
    static constexpr int B_KFULL = B_QEMPTY + QBUF;
    static constexpr int B_KEMPTY = B_KFULL + STK;
    static constexpr int B_VFULL = B_KEMPTY + STK;
    static constexpr int B_VEMPTY = B_VFULL + STV;
    static constexpr int B_SFULL = B_VEMPTY + STV;      // [2] S' buffer written
    static constexpr int B_PFULL = B_SFULL + 2;         // [2] P' buffer written (one arrival per softmax warp)
    static constexpr int B_PVDONE = B_PFULL + 2;        // [2] PV' that read P' buffer b completed
    static constexpr int B_OFREE = B_PVDONE + 2;        // [2] epilogue has read O' buffer b and its row stats
    static constexpr int B_STATS = B_OFREE + 2;         // [2] softmax has written the row stats of buffer b
    static constexpr int B_SEGPV = B_STATS + 2;         // [2] a segment's last PV' into O' buffer b completed
    static constexpr int B_RED = B_SEGPV + 2;           // softmax warps: per-tile row reductions
    static constexpr int B_XSYNC = B_RED + 1;           // softmax warps: epilogue / merge steps (FP8)
    static constexpr int B_ESYNC = B_XSYNC + 1;         // epilogue warps: epilogue / merge steps
    static constexpr int B_FINAL = B_ESYNC + 1;
    static constexpr int B_KCONV = B_FINAL + 1;         // [STK] FP8: K stage widened to f16
    static constexpr int B_VCONV = B_KCONV + STK;       // [STV] FP8: V stage widened to f16
    static constexpr int B_QCONV = B_VCONV + STV;       // [QBUF] FP8: Q buffer converted to f16
    static constexpr int B_BOUNDS = B_QCONV + QBUF;     // the span bounds table is filled
    static constexpr int NBAR = B_BOUNDS + 1;
    // the control block holds float4-read arrays: 128-byte aligned whatever NBAR is
    static constexpr int OFF_MISC = (OFF_BAR + NBAR * 8 + 127) & ~127;
    static_assert(OFF_MISC % 128 == 0, "control block alignment");
    static constexpr int MISC_BYTES = 1536 + 4 * (kMaxGrid + 1) + 4 * (kMaxWeightedB + 1) + 4 * kMaxWeightedB;
    static constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t TM_COLS = 64;
    static constexpr uint32_t TM_S = 0;   // + 16 * buffer
    __host__ __device__ static constexpr uint32_t tm_o(int b) { return 32u + 16u * static_cast<uint32_t>(b); }
    static constexpr uint32_t IDESC_S =
        FP8 ? ptx::umma_idesc_f16_f32(BN, DEC_NQ, false, false) : ptx::umma_idesc_bf16_f32(BN, DEC_NQ, false, false);
    static constexpr uint32_t IDESC_PV =
        FP8 ? ptx::umma_idesc_f16_f32(D, DEC_NQ, true, false) : ptx::umma_idesc_bf16_f32(D, DEC_NQ, true, false);
    // FP8: the raw E4M3 tile (128 keys x 128 bytes, 128-byte swizzle) lands in the
    // upper half of its stage; widened, it fills the stage as two 64-column f16 boxes
    static constexpr int KV_RAW_OFF = FP8 ? KV_BOX : 0;
    static constexpr int RAW_TILE = BN * 128;
    // the stages a role waits for before an MMA reads them
    static constexpr int B_KREADY = FP8 ? B_KCONV : B_KFULL;
    static constexpr int B_VREADY = FP8 ? B_VCONV : B_VFULL;
    static constexpr int B_QREADY = FP8 ? B_QCONV : B_QFULL;
};

// Two E4M3 bytes (the first in the low byte) -> two f16 (the first in the low half).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
    return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// FP8: widen one stage in place, 128 converter threads (ct = 0..127).  Raw byte
// chunk c (16 keys' worth of columns 16c..16c+15) of row r sits at r*128 +
// ((c ^ r%8) << 4) of the raw tile; its 16 f16 go to box c/4, chunks 2(c%4) and
// 2(c%4)+1 of row r.  Box 1 overlaps the raw tile row for row, so each warp
// reads its four rows completely before it writes them.  Rows >= zrow are
// written as zeros.
template <class C>
__device__ __forceinline__ void dec_widen_stage(uint8_t* stage, int ct, int zrow) {
    const uint8_t* raw = stage + C::KV_RAW_OFF;
#pragma unroll 2
    for (int k = 0; k < (C::BN * 8) / 128; ++k) {
        const int i = ct + 128 * k;
        const int r = i >> 3, c = i & 7;
        const uint4 x = *reinterpret_cast<const uint4*>(raw + r * 128 + ((c ^ (r & 7)) << 4));
        __syncwarp();
        uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
        if (r < zrow) {
            lo = make_uint4(e4m3x2_to_f16x2(x.x), e4m3x2_to_f16x2(x.x >> 16), e4m3x2_to_f16x2(x.y),
                            e4m3x2_to_f16x2(x.y >> 16));
            hi = make_uint4(e4m3x2_to_f16x2(x.z), e4m3x2_to_f16x2(x.z >> 16), e4m3x2_to_f16x2(x.w),
                            e4m3x2_to_f16x2(x.w >> 16));
        }
        uint8_t* row = stage + (c >> 2) * C::KV_BOX + r * 128;
        const int c2 = 2 * (c & 3);
        *reinterpret_cast<uint4*>(row + ((c2 ^ (r & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(row + (((c2 + 1) ^ (r & 7)) << 4)) = hi;
        __syncwarp();
    }
}

struct DecMisc {
    uint32_t tmem_base;       // the first four fields match Misc (bounded waits read abort)
    volatile int abort;
    volatile int merge_flag;
    int pad;
    SpanStart span;
    float red[2][DEC_NQ][4];  // per-tile row reductions: [phase][row][softmax warp]
    float mlse[DEC_NQ];       // merged lse per packed row (in-kernel merge)
    int nmerge;
    int mslot[kMaxMergeSlots];
    float seg_w[2][DEC_NQ];   // per row of the segment in O' buffer b: the factor O' is scaled by
    float seg_lse[2][DEC_NQ]; //   and the row's (or the piece's) lse
    int etk;                  // the epilogue's split piece completed its row-block (it merges)
    int bounds[kMaxGrid + 1];  // flat start of every CTA's span (cost-weighted), bounds[NC] = tot
    int yb[kMaxWeightedB + 1]; // weighted start of every batch (the plan's table)
    int lens[kMaxWeightedB];   // every batch's logical length (the plan's reads, kept for the walkers)
};

// Reduce NR per-thread values over the 32 lanes of a warp, one row per lane group:
// returns the reduction of row dec_row_of<NR>(lane).  Each halving step trades the
// half a lane does not keep with its partner, so 2*NR - 1 shuffles in all.
template <int NR, bool MAX>
__device__ __forceinline__ float dec_warp_reduce(const float (&x)[NR], int lane) {
    float v[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) v[i] = x[i];
    int bit = 16;
#pragma unroll
    for (int step = NR / 2; step >= 1; step /= 2, bit >>= 1) {
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < step; ++i) {
            const float keep = up ? v[i + step] : v[i];
            const float send = up ? v[i] : v[i + step];
            const float got = __shfl_xor_sync(0xffffffffu, send, bit);
            v[i] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
#pragma unroll
    for (int b = bit; b >= 1; b >>= 1) {
        const float got = __shfl_xor_sync(0xffffffffu, v[0], b);
        v[0] = MAX ? fmaxf(v[0], got) : v[0] + got;
    }
    return v[0];
}
template <int NR>
__device__ __forceinline__ int dec_row_of(int lane) {
    return (NR == 8) ? (((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1))
                     : (((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1));
}
template <int NR>
__device__ __forceinline__ bool dec_row_writer(int lane) {
    return (NR == 8) ? (lane & 3) == 0 : (lane & 1) == 0;
}

// O' (+)= V(gg)^T P'(gg): A = the V tile read MN-major (M = head dims), B = P'^T
// (K-major).  Not inlined: the MMA thread reaches it from three places, and one
// shared copy is in the instruction cache after the first tile (a copy that first
// runs at a segment switch would be fetched while every SM streams K/V).
template <class C>
__device__ __noinline__ bool dec_issue_pv(const Params& p, Misc* wmisc, uint32_t bar0, uint32_t sbase, uint32_t tmem,
                                          uint32_t gg, bool first, int seg, bool last) {
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
    const int st = gg % C::STV;
    const int ob = seg & 1;
    if (!wait_bar(bar(C::B_PFULL + (gg & 1u)), (gg >> 1) & 1u, wmisc, p)) return false;
    if (!wait_bar(bar(C::B_VREADY + st), (gg / C::STV) & 1u, wmisc, p)) return false;
    // a segment's first PV' overwrites O' buffer seg % 2: its epilogue two segments back must have read it
    if (first && seg >= 2 && !wait_bar(bar(C::B_OFREE + ob), ((seg - 2) >> 1) & 1, wmisc, p)) return false;
    ptx::tc_fence_after();
    const uint32_t vbase = sbase + C::OFF_V + st * C::KV_BYTES;
    const uint32_t pbase = sbase + C::OFF_P + (gg & 1u) * C::P_BYTES;
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk) {
        const uint64_t ad = ptx::umma_desc_sw128(vbase + kk * 2048, C::KV_BOX, 1024);
        const uint64_t bd = ptx::umma_desc_sw128(pbase + (kk >> 2) * C::P_BOX + (kk & 3) * 32, 16, 1024);
        ptx::umma_bf16_ss(tmem + C::tm_o(ob), ad, bd, C::IDESC_PV, (kk > 0 || !first) ? 1u : 0u);
    }
    ptx::umma_commit(bar(C::B_PVDONE + (gg & 1u)));
    ptx::umma_commit(bar(C::B_VEMPTY + st));
    if (last) ptx::umma_commit(bar(C::B_SEGPV + ob));
    return true;
}

template <class C>
__global__ void __launch_bounds__(C::NTHREADS, 1)
gqa_dec_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Params p) {
    constexpr int NR = C::NR;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw;
    const uint32_t sbase = ptx::smem_addr(smem);
    if (sbase & 1023u) {  // the swizzled tiles need a 1024-aligned window
        if (threadIdx.x == 0) atomicCAS(p.err, 0, DEV_ERR_SMEM_ALIGN);
        return;
    }
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
    DecMisc* misc = reinterpret_cast<DecMisc*>(smem + C::OFF_MISC);
    Misc* wmisc = reinterpret_cast<Misc*>(misc);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const int NC = gridDim.x;

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::QBUF; ++i) {
            ptx::mbar_init(bar(C::B_QFULL + i), 1);
            ptx::mbar_init(bar(C::B_QEMPTY + i), 1);
        }
        for (int i = 0; i < C::STK; ++i) {
            ptx::mbar_init(bar(C::B_KFULL + i), 1);
            ptx::mbar_init(bar(C::B_KEMPTY + i), 1);
        }
        for (int i = 0; i < C::STV; ++i) {
            ptx::mbar_init(bar(C::B_VFULL + i), 1);
            ptx::mbar_init(bar(C::B_VEMPTY + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(C::B_SFULL + i), 1);
            ptx::mbar_init(bar(C::B_PFULL + i), 4);
            ptx::mbar_init(bar(C::B_PVDONE + i), 1);
            ptx::mbar_init(bar(C::B_OFREE + i), 4);  // one arrival per epilogue warp
            ptx::mbar_init(bar(C::B_STATS + i), 4);  // one arrival per softmax warp
            ptx::mbar_init(bar(C::B_SEGPV + i), 1);
        }
        for (int i = 0; i < C::STK; ++i) ptx::mbar_init(bar(C::B_KCONV + i), 4);
        for (int i = 0; i < C::STV; ++i) ptx::mbar_init(bar(C::B_VCONV + i), 4);
        for (int i = 0; i < C::QBUF; ++i) ptx::mbar_init(bar(C::B_QCONV + i), 4);
        ptx::mbar_init(bar(C::B_BOUNDS), 1);
        ptx::mbar_init(bar(C::B_RED), 4);
        ptx::mbar_init(bar(C::B_XSYNC), 4);
        ptx::mbar_init(bar(C::B_ESYNC), 4);
        ptx::mbar_init(bar(C::B_FINAL), 1);
        misc->abort = 0;
        misc->merge_flag = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tm_q);
        ptx::tma_prefetch_desc(&tm_k);
        ptx::tma_prefetch_desc(&tm_v);
    }
    if (warp == 2) {
        ptx::tmem_alloc(ptx::smem_addr(&misc->tmem_base), C::TM_COLS);
        ptx::tmem_relinquish();
    }
    if (warp == 0) {
        if (p.B <= kMaxWeightedB) plan_span_weighted(p, cta, NC, &misc->span, misc->yb, misc->lens);
        else plan_span(p, cta, NC, &misc->span);  // equal spans (the host sets seg_w = 0)
    }
    if (warp >= 4 && warp < 8) {
        // P' rows past NR are never written by the softmax: keep them zero
        uint4* pz = reinterpret_cast<uint4*>(smem + C::OFF_P);
        for (int i = threadIdx.x - 128; i < 2 * C::P_BYTES / 16; i += NSOFT_DEC) pz[i] = make_uint4(0, 0, 0, 0);
        ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before();
    __syncwarp();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    // The epilogue of segment seg_i, by four warps (warp q reads TMEM lane
    // quadrant q; thread et = 32q + lane owns head dim et): O'(seg_i % 2) times
    // 1/l written as the output rows (a direct segment) or as a split piece; a
    // piece then takes the row-block's ticket, and the piece that completes the
    // row-block merges all of its pieces.  `sync` is the four warps' bounded
    // barrier.  The row loops are rolled: this code first runs while every SM
    // streams K/V, and each of its instruction-cache lines is fetched then.
    auto epi_segment = [&](const Seg& sg, int seg_i, int q, auto&& sync) -> bool {
        const int ob = seg_i & 1;
        const int et = q * 32 + lane;
        const int kl = et;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        bool ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_STATS + ob), (seg_i >> 1) & 1, wmisc, p));
        if (ok) ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_SEGPV + ob), (seg_i >> 1) & 1, wmisc, p));
        if (!ok) return false;
        ptx::tc_fence_after();
        const RB rb = rb_of(p, sg.w);
        uint32_t o[NR];
        {
            const uint32_t to = tmem + lane_off + C::tm_o(ob);
            if constexpr (NR == 16) ptx::tmem_ld16(to, o);
            else ptx::tmem_ld8(to, o);
            ptx::tmem_wait_ld();
        }
        float w[NR], lse_r[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            w[r] = misc->seg_w[ob][r];
            lse_r[r] = misc->seg_lse[ob][r];
        }
        // O'(ob) and the row factors are read: the segment after next may use them
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(C::B_OFREE + ob));
        const bool direct = (sg.kind == 0);
        if (direct) {
#pragma unroll
            for (int r = 0; r < NR; ++r)
                if (r < rb.rows_valid) {
                    const long long fr = rb.q_row0 + r;  // flat row (b*Hq + h)*Tq + i
                    p.out[fr * C::D + kl] = __float2bfloat16_rn(w[r] != 0.f ? __uint_as_float(o[r]) * w[r] : 0.f);
                    if (kl == 0 && p.lse != nullptr) p.lse[fr] = lse_r[r];
                }
        } else {
#pragma unroll
            for (int r = 0; r < NR; ++r)
                if (r < rb.rows_valid) {
                    const long long prow = static_cast<long long>(sg.slot) * BM + r;
                    __stcg(p.part_o + prow * C::D + kl, w[r] != 0.f ? __uint_as_float(o[r]) * w[r] : 0.f);
                    if (kl == 0) __stcg(p.part_lse + prow, lse_r[r]);
                }
            // release: this thread's partial rows are visible GPU-wide before the ticket
            __threadfence();
        }
        if (direct) return true;
        // a split piece: once all of its rows are written, count it on the
        // row-block's ticket (release fence, then the atomic)
        if (!sync()) return false;
        if (et == 0) {
            int tk = 0;
            if (wait_bar(bar(C::B_BOUNDS), 0, wmisc, p)) {
                const int* bd = misc->bounds;
                const int c_first = cta_of_table(bd, NC, sg.pw);
                const int c_last = cta_of_table(bd, NC, sg.pw + sg.ntiles - 1);
                int ncontrib = 0;
                for (int cc = c_first; cc <= c_last; ++cc) ncontrib += bd[cc] < bd[cc + 1];
                const int old = atomicAdd(p.counters + sg.w, 1);
                tk = (old == ncontrib - 1);
            }
            misc->etk = tk;
        }
        if (!sync() || misc->abort) return false;
        if (!misc->etk) return true;
        // this piece completed the row-block: merge every piece's rows
        __threadfence();
        const int* bd = misc->bounds;
        const int c_first = cta_of_table(bd, NC, sg.pw);
        const int c_last = cta_of_table(bd, NC, sg.pw + sg.ntiles - 1);
        const bool c0_first = bd[c_first] == sg.pw;
        const long long RW = BM;
        if (q == 0) {
            int nm = 0;
            for (int base = c_first; base <= c_last; base += 32) {
                const int cc = base + lane;
                const bool has = cc <= c_last && bd[cc] < bd[cc + 1];
                const unsigned m = __ballot_sync(0xffffffffu, has);
                const int k = nm + __popc(m & ((1u << lane) - 1u));
                if (has && k < kMaxMergeSlots) misc->mslot[k] = static_cast<int>(merge_slot(cc, c_first, c0_first));
                nm += __popc(m);
            }
            if (lane == 0) misc->nmerge = nm;
        }
        if (!sync()) return false;
        const int nm = misc->nmerge;
        auto slot_of = [&](int k) -> long long {  // k-th contributing CTA's slot
            if (nm <= kMaxMergeSlots) return misc->mslot[k];
            int seen = 0;
            for (int cc = c_first; cc <= c_last; ++cc) {
                if (!(bd[cc] < bd[cc + 1])) continue;
                if (seen++ == k) return merge_slot(cc, c_first, c0_first);
            }
            return 0;
        };
        // lse of each merged row (the sink enters here, once); eight pieces' loads at a time
        for (int r = et; r < rb.rows_valid; r += 128) {
            const int hr = rb.g * p.G + r / p.Tq;
            const float sk = (p.sink != nullptr) ? __ldg(p.sink + hr) : -INFINITY;
            float Lx = sk, z = 0.f;
            for (int k0 = 0; k0 < nm; k0 += 8) {
                float lv[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    lv[jj] = (k0 + jj < nm) ? __ldcg(p.part_lse + slot_of(k0 + jj) * RW + r) : -INFINITY;
                float mx = Lx;
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) mx = fmax_nan(mx, lv[jj]);
                if (mx != -INFINITY) {
                    // running (max, sum) over the pieces seen so far
                    z = (Lx != -INFINITY) ? z * __expf(Lx - mx) : 0.f;
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) z += __expf(lv[jj] - mx);
                    Lx = mx;
                }
            }
            float ltr = -INFINITY;
            if (Lx != -INFINITY) {
                if (sk != -INFINITY) z += __expf(sk - Lx);
                ltr = Lx + __logf(z);
            }
            misc->mlse[r] = ltr;
            if (p.lse != nullptr) p.lse[rb.q_row0 + r] = ltr;
        }
        if (!sync()) return false;
        // O rows: weight exp(lse_k - lse) per piece; thread = head dim; every
        // row's loads of two pieces in flight together
        float lt[NR], acc[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            lt[r] = (r < rb.rows_valid) ? misc->mlse[r] : -INFINITY;
            acc[r] = 0.f;
        }
        for (int k0 = 0; k0 < nm; k0 += 2) {
            float lw[2][NR], xv[2][NR];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const bool has = k0 + jj < nm;
                const long long sl = has ? slot_of(k0 + jj) : 0;
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const bool live = has && lt[r] != -INFINITY;
                    lw[jj][r] = live ? __ldcg(p.part_lse + sl * RW + r) : -INFINITY;
                    xv[jj][r] = live ? __ldcg(p.part_o + (sl * RW + r) * C::D + kl) : 0.f;
                }
            }
#pragma unroll
            for (int jj = 0; jj < 2; ++jj)
#pragma unroll
                for (int r = 0; r < NR; ++r)
                    if (lw[jj][r] != -INFINITY) acc[r] += __expf(lw[jj][r] - lt[r]) * xv[jj][r];
        }
#pragma unroll
        for (int r = 0; r < NR; ++r)
            if (r < rb.rows_valid) p.out[(rb.q_row0 + r) * C::D + kl] = __float2bfloat16_rn(acc[r]);
        if (et == 0) p.counters[sg.w] = 0;
        // the shared merge fields are free again once every thread is past them
        return sync();
    };

    if (warp < 4) {
        // ------------------------------------------------------------ Q / K producer
        if (warp == 0 && lane == 0) {
            const uint64_t pol_q = ptx::policy_evict_last();
            const uint64_t pol_kv = ptx::policy_evict_first();
            SegWalker wk;
            wk.init(p, misc->span, cta, p.B <= kMaxWeightedB ? misc->lens : nullptr);
            Seg sg;
            int seg_i = 0;
            uint32_t g = 0;
            bool ok = true;
            uint32_t k_issued[C::STK], q_issued[C::QBUF];
            for (int i = 0; i < C::STK; ++i) k_issued[i] = 0;
            for (int i = 0; i < C::QBUF; ++i) q_issued[i] = 0;
            while (ok && wk.next(p, sg)) {
                if (sg.t1 <= sg.t0) continue;
                const RB rb = rb_of(p, sg.w);
                const int qb = seg_i % C::QBUF;
                ok = wait_bar(bar(C::B_QEMPTY + qb), ((seg_i / C::QBUF) & 1) ^ 1, wmisc, p);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(bar(C::B_QFULL + qb), C::NBOX * p.q_box_rows * 128);
                ++q_issued[qb];
                for (int bx = 0; bx < C::NBOX; ++bx)
                    ptx::tma_load_2d(sbase + C::OFF_Q + qb * C::Q_BYTES + bx * C::Q_BOX, &tm_q, bx * 64,
                                     static_cast<int>(rb.q_row0), bar(C::B_QFULL + qb), pol_q);
                for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                    const int st = g % C::STK;
                    ok = wait_bar(bar(C::B_KEMPTY + st), ((g / C::STK) & 1) ^ 1, wmisc, p);
                    if (!ok) break;
                    ++k_issued[st];
                    if constexpr (C::FP8) {
                        ptx::mbar_arrive_expect_tx(bar(C::B_KFULL + st), p.kv_box_rows * 128);
                        ptx::tma_load_2d(sbase + C::OFF_K + st * C::KV_BYTES + C::KV_RAW_OFF, &tm_k, 0,
                                         static_cast<int>(rb.kv_row0 + static_cast<long long>(t) * C::BN),
                                         bar(C::B_KFULL + st), pol_kv);
                    } else {
                        load_kv_tile<C>(p, &tm_k, sbase + C::OFF_K + st * C::KV_BYTES, bar(C::B_KFULL + st), rb, t,
                                        sg.n, pol_kv);
                    }
                }
                ++seg_i;
            }
            for (int i = 0; i < C::STK; ++i) drain_bar(bar(C::B_KFULL + i), k_issued[i], p.timeout_cycles);
            for (int i = 0; i < C::QBUF; ++i) drain_bar(bar(C::B_QFULL + i), q_issued[i], p.timeout_cycles);
        }
        // ------------------------------------------------------------ V producer
        else if (warp == 1 && lane == 0) {
            const uint64_t pol_kv = ptx::policy_evict_first();
            SegWalker wk;
            wk.init(p, misc->span, cta, p.B <= kMaxWeightedB ? misc->lens : nullptr);
            Seg sg;
            uint32_t g = 0;
            bool ok = true;
            uint32_t v_issued[C::STV];
            for (int i = 0; i < C::STV; ++i) v_issued[i] = 0;
            while (ok && wk.next(p, sg)) {
                if (sg.t1 <= sg.t0) continue;
                const RB rb = rb_of(p, sg.w);
                for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                    const int st = g % C::STV;
                    ok = wait_bar(bar(C::B_VEMPTY + st), ((g / C::STV) & 1) ^ 1, wmisc, p);
                    if (!ok) break;
                    ++v_issued[st];
                    if constexpr (C::FP8) {
                        ptx::mbar_arrive_expect_tx(bar(C::B_VFULL + st), p.kv_box_rows * 128);
                        ptx::tma_load_2d(sbase + C::OFF_V + st * C::KV_BYTES + C::KV_RAW_OFF, &tm_v, 0,
                                         static_cast<int>(rb.kv_row0 + static_cast<long long>(t) * C::BN),
                                         bar(C::B_VFULL + st), pol_kv);
                    } else {
                        load_kv_tile<C>(p, &tm_v, sbase + C::OFF_V + st * C::KV_BYTES, bar(C::B_VFULL + st), rb, t,
                                        sg.n, pol_kv);
                    }
                }
            }
            for (int i = 0; i < C::STV; ++i) drain_bar(bar(C::B_VFULL + i), v_issued[i], p.timeout_cycles);
        }
        // ------------------------------------------------------------ MMA issuer
        else if (warp == 2 && lane == 0) {
            SegWalker wk;
            wk.init(p, misc->span, cta, p.B <= kMaxWeightedB ? misc->lens : nullptr);
            Seg sg;
            int seg_i = 0;
            uint32_t g = 0;
            bool ok = true;
            // S'(g) = K(g) Q^T: A = the K tile (M = keys, K-major), B = the 16-row Q tile (K-major)
            auto issue_s = [&](uint32_t gg, uint32_t qbase, uint32_t kbase) {
                const uint32_t d = tmem + C::TM_S + 16u * (gg & 1u);
#pragma unroll
                for (int kk = 0; kk < C::D / 16; ++kk) {
                    const uint32_t off = (kk & 3) * 32;
                    const uint64_t ad = ptx::umma_desc_sw128(kbase + (kk >> 2) * C::KV_BOX + off, 16, 1024);
                    const uint64_t bd = ptx::umma_desc_sw128(qbase + (kk >> 2) * C::Q_BOX + off, 16, 1024);
                    ptx::umma_bf16_ss(d, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
                }
                ptx::umma_commit(bar(C::B_SFULL + (gg & 1u)));
            };
            // O' (+)= V(gg)^T P'(gg): A = the V tile read MN-major (M = head dims), B = P'^T (K-major)
            auto issue_pv = [&](uint32_t gg, bool first, int seg, bool last) -> bool {
                return dec_issue_pv<C>(p, wmisc, bar0, sbase, tmem, gg, first, seg, last);
            };
            bool have_prev = false, prev_first = false;
            uint32_t prev_g = 0;
            int prev_seg = 0;
            while (ok && wk.next(p, sg)) {
                if (sg.t1 <= sg.t0) continue;
                // the previous segment's last PV' goes out before this segment's Q is awaited
                if (have_prev) {
                    ok = issue_pv(prev_g, prev_first, prev_seg, true);
                    if (!ok) break;
                    have_prev = false;
                }
                const int qb = seg_i % C::QBUF;
                ok = wait_bar(bar(C::B_QREADY + qb), (seg_i / C::QBUF) & 1, wmisc, p);
                if (!ok) break;
                const uint32_t qbase = sbase + C::OFF_Q + qb * C::Q_BYTES;
                for (int t = sg.t0; t < sg.t1 && ok; ++t, ++g) {
                    const int stk = g % C::STK;
                    ok = wait_bar(bar(C::B_KREADY + stk), (g / C::STK) & 1, wmisc, p);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    issue_s(g, qbase, sbase + C::OFF_K + stk * C::KV_BYTES);
                    ptx::umma_commit(bar(C::B_KEMPTY + stk));
                    if (t == sg.t1 - 1) ptx::umma_commit(bar(C::B_QEMPTY + qb));
                    if (have_prev) {
                        ok = issue_pv(prev_g, prev_first, prev_seg, false);
                        if (!ok) break;
                    }
                    have_prev = true;
                    prev_g = g;
                    prev_first = (t == sg.t0);
                    prev_seg = seg_i;
                }
                ++seg_i;
            }
            if (ok && have_prev) ok = issue_pv(prev_g, prev_first, prev_seg, true);
            ptx::umma_commit(bar(C::B_FINAL));
            drain_bar(bar(C::B_FINAL), 1, p.timeout_cycles);
        }
        // ------------------------------------------------------------ span bounds
        else if (warp == 3) {
            // the whole warp fills the span bounds of every CTA (the tickets and the
            // merges look other CTAs' spans up there)
            if (p.B <= kMaxWeightedB) {
                fill_span_bounds(p, misc->yb, NC, misc->bounds);
            } else {
                for (int k = lane; k <= NC; k += 32)
                    misc->bounds[k] = static_cast<int>(span_begin(k, misc->span.tot, NC));
                __syncwarp();
            }
            if (lane == 0) ptx::mbar_arrive(bar(C::B_BOUNDS));
        }
    }
    // ---------------------------------------------------------------- softmax warps
    else if (warp < 8) {
        const int quad = warp & 3;
        const int kl = quad * 32 + lane;  // key of the tile = S' lane; head dim = O' lane
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const int stid = threadIdx.x - 128;
        uint32_t rph = 0, xph = 0;
        auto xsync = [&]() -> bool {  // the four softmax warps, bounded
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(C::B_XSYNC));
            const bool r = wait_bar(bar(C::B_XSYNC), xph & 1, wmisc, p);
            ++xph;
            ptx::tc_fence_after();
            return __all_sync(0xffffffffu, r);
        };
        // reduce NR values per thread over all 128 keys of the softmax warps
        auto cta_reduce = [&](const float (&x)[NR], float (&out)[NR], bool is_max) -> bool {
            const float wv = is_max ? dec_warp_reduce<NR, true>(x, lane) : dec_warp_reduce<NR, false>(x, lane);
            float(*red)[4] = misc->red[rph & 1];
            if (dec_row_writer<NR>(lane)) red[dec_row_of<NR>(lane)][quad] = wv;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(C::B_RED));
            bool okr = wait_bar(bar(C::B_RED), rph & 1, wmisc, p);
            ++rph;
            okr = __all_sync(0xffffffffu, okr);
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                const float4 w4 = *reinterpret_cast<const float4*>(&red[r][0]);
                out[r] = is_max ? fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w)) : (w4.x + w4.y) + (w4.z + w4.w);
            }
            return okr;
        };
        SegWalker wk;
        wk.init(p, misc->span, cta, p.B <= kMaxWeightedB ? misc->lens : nullptr);
        Seg sg;
        uint32_t g = 0;
        bool ok = true;
        int seg_i = 0;
        // P'^T address of this thread's key in a P' buffer: row r adds r*128 and
        // swizzles the 16-byte chunk by r % 8
        const int pkey_box = kl >> 6, pkey_chunk = (kl & 63) >> 3, pkey_in = (kl & 7) * 2;

        while (ok && wk.next(p, sg)) {
            if (sg.t1 <= sg.t0) continue;
            const RB rb = rb_of(p, sg.w);
            // visible keys of each packed row: key <= lim[r] (-1: row absent)
            int lim[NR];
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                int l = -1;
                if (r < rb.rows_valid) {
                    const int i = r % p.Tq;
                    l = p.causal ? (sg.n - p.Tq + i) : (sg.n - 1);
                    if (l > sg.n - 1) l = sg.n - 1;
                }
                lim[r] = l;
            }
            float m_run[NR], l_t[NR];
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                m_run[r] = -INFINITY;
                l_t[r] = 0.f;
            }
            for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                const bool first = (t == sg.t0);
                ok = wait_bar(bar(C::B_SFULL + (g & 1u)), (g >> 1) & 1u, wmisc, p);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ptx::tc_fence_after();
                float x[NR];
                {
                    uint32_t sr[NR];
                    const uint32_t ts = tmem + lane_off + C::TM_S + 16u * (g & 1u);
                    if constexpr (NR == 16) ptx::tmem_ld16(ts, sr);
                    else ptx::tmem_ld8(ts, sr);
                    ptx::tmem_wait_ld();
                    const int key = t * C::BN + kl;
                    // mask by selection (never by adding -inf: NaN + -inf stays NaN)
#pragma unroll
                    for (int r = 0; r < NR; ++r) x[r] = (key <= lim[r]) ? __uint_as_float(sr[r]) * p.scale_log2 : -INFINITY;
                }
                float mt[NR];
                ok = cta_reduce(x, mt, true);
                if (!ok) break;
                // online softmax with a lazy rescale: the reference max moves only
                // when a row's max grows by more than 2^8
                bool grow = false;
#pragma unroll
                for (int r = 0; r < NR; ++r) grow |= mt[r] > m_run[r] + RESCALE_THRESHOLD;
                if (grow) {
                    float alpha[NR];
#pragma unroll
                    for (int r = 0; r < NR; ++r) {
                        const float mn = fmaxf(m_run[r], mt[r]);
                        alpha[r] = (m_run[r] == -INFINITY) ? 0.f : ptx::ex2(m_run[r] - mn);
                        l_t[r] *= alpha[r];
                        m_run[r] = mn;
                    }
                    if (!first) {
                        // O' holds PV'(g-1) once it completes; scale column r by alpha[r]
                        bool okw = wait_bar(bar(C::B_PVDONE + ((g - 1) & 1u)), ((g - 1) >> 1) & 1u, wmisc, p);
                        okw = __all_sync(0xffffffffu, okw);
                        if (!okw) { ok = false; break; }
                        ptx::tc_fence_after();
                        const uint32_t to = tmem + lane_off + C::tm_o(seg_i & 1);
                        uint32_t o[NR];
                        if constexpr (NR == 16) ptx::tmem_ld16(to, o);
                        else ptx::tmem_ld8(to, o);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int r = 0; r < NR; ++r) o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha[r]);
                        if constexpr (NR == 16) ptx::tmem_st16(to, o);
                        else ptx::tmem_st8(to, o);
                        ptx::tmem_wait_st();
                    }
                }
                // P' buffer g % 2 was last read by PV'(g-2)
                if (g >= 2) {
                    bool okw = wait_bar(bar(C::B_PVDONE + (g & 1u)), ((g - 2) >> 1) & 1u, wmisc, p);
                    okw = __all_sync(0xffffffffu, okw);
                    if (!okw) { ok = false; break; }
                }
                uint8_t* pb = smem + C::OFF_P + (g & 1u) * C::P_BYTES + pkey_box * C::P_BOX + pkey_in;
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const float mu = (m_run[r] == -INFINITY) ? 0.f : m_run[r];
                    const float pr = ptx::ex2(x[r] - mu);
                    l_t[r] += pr;
                    if constexpr (C::FP8)
                        *reinterpret_cast<__half*>(pb + r * 128 + ((pkey_chunk ^ (r & 7)) << 4)) = __float2half_rn(pr);
                    else
                        *reinterpret_cast<__nv_bfloat16*>(pb + r * 128 + ((pkey_chunk ^ (r & 7)) << 4)) = __float2bfloat16_rn(pr);
                }
                // padded key rows of the V tile reach the MMA as zeros (0 * NaN = NaN);
                // with FP8 K/V the converter warps write them as zeros
                if (!C::FP8 && (t + 1) * C::BN > sg.n) {
                    const int st = g % C::STV;
                    bool okv = wait_bar(bar(C::B_VFULL + st), (g / C::STV) & 1, wmisc, p);
                    okv = __all_sync(0xffffffffu, okv);
                    if (!okv) { ok = false; break; }
                    if (t * C::BN + kl >= sg.n) {
                        uint8_t* vt = smem + C::OFF_V + st * C::KV_BYTES + kl * 128;
#pragma unroll
                        for (int bx = 0; bx < C::NBOX; ++bx)
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                *reinterpret_cast<uint4*>(vt + bx * C::KV_BOX + c * 16) = make_uint4(0, 0, 0, 0);
                    }
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::B_PFULL + (g & 1u)));
            }
            if (!ok) break;

            // ------------------------------------------------ segment end
            // The row statistics go to shared memory; the epilogue (the epilogue
            // warps, or these warps with FP8 K/V) finishes the segment from O'(seg % 2).
            {
                float lsum[NR];
                ok = cta_reduce(l_t, lsum, false);
                if (!ok) break;
                const int ob = seg_i & 1;
                // the epilogue of the segment two back has read this statistics slot
                if (seg_i >= 2) {
                    ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_OFREE + ob), ((seg_i - 2) >> 1) & 1, wmisc, p));
                    if (!ok) break;
                }
                // thread r < NR finishes row r: the factor O' is scaled by and the lse
                // (with the sink for a direct segment; a split piece's own lse otherwise)
                if (stid < NR) {
                    float mr = 0.f, lr = 0.f;
#pragma unroll
                    for (int r = 0; r < NR; ++r)
                        if (stid == r) {
                            mr = m_run[r];
                            lr = lsum[r];
                        }
                    float w = 0.f, lse_v = -INFINITY;
                    if (stid < rb.rows_valid) {
                        if (sg.kind == 0) {
                            const int h = rb.g * p.G + stid / p.Tq;
                            const float sk = (p.sink != nullptr) ? __ldg(p.sink + h) * LOG2E : -INFINITY;
                            const float M = fmax_nan(mr, sk);
                            if (M != -INFINITY) {
                                const float a = pos_or_nan(lr) ? ptx::ex2(mr - M) : 0.f;
                                const float lt = lr * a + ((sk != -INFINITY) ? ptx::ex2(sk - M) : 0.f);
                                if (pos_or_nan(lt)) {
                                    w = a / lt * p.v_scale;
                                    lse_v = (M + __log2f(lt)) * LN2;
                                }
                            }
                        } else if (pos_or_nan(lr)) {
                            w = p.v_scale / lr;
                            lse_v = (mr + __log2f(lr)) * LN2;
                        }
                    }
                    misc->seg_w[ob][stid] = w;
                    misc->seg_lse[ob][stid] = lse_v;
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::B_STATS + ob));
            }
            if constexpr (!C::EPIW) {
                ok = epi_segment(sg, seg_i, quad, xsync);
                if (!ok) break;
            }
            ++seg_i;
        }
    }
    // ---------------------------------------------------------------- epilogue warps
    else if constexpr (C::EPIW) {
        const int quad = warp & 3;
        uint32_t eph = 0;
        auto esync = [&]() -> bool {  // the four epilogue warps, bounded
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(C::B_ESYNC));
            const bool r = wait_bar(bar(C::B_ESYNC), eph & 1, wmisc, p);
            ++eph;
            ptx::tc_fence_after();
            return __all_sync(0xffffffffu, r);
        };
        SegWalker wk;
        wk.init(p, misc->span, cta, p.B <= kMaxWeightedB ? misc->lens : nullptr);
        Seg sg;
        int seg_i = 0;
        bool ok = true;
        while (ok && wk.next(p, sg)) {
            if (sg.t1 <= sg.t0) continue;
            ok = epi_segment(sg, seg_i, quad, esync);
            ++seg_i;
        }
    }

    // ---------------------------------------------------------------- FP8 converter warps
    else if constexpr (C::FP8) {
        const int ct = threadIdx.x - 256;  // 0..127
        SegWalker wk;
        wk.init(p, misc->span, cta, p.B <= kMaxWeightedB ? misc->lens : nullptr);
        Seg sg;
        int seg_i = 0;
        uint32_t g = 0;
        bool ok = true;
        while (ok && wk.next(p, sg)) {
            if (sg.t1 <= sg.t0) continue;
            // Q: bf16 -> f16 in place (same layout)
            const int qb = seg_i % C::QBUF;
            ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_QFULL + qb), (seg_i / C::QBUF) & 1, wmisc, p));
            if (!ok) break;
            uint4* qv = reinterpret_cast<uint4*>(smem + C::OFF_Q + qb * C::Q_BYTES);
            for (int i = ct; i < C::Q_BYTES / 16; i += 128) {
                uint4 x = qv[i];
                uint32_t* w4 = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[j]));
                    const __half2 h = __floats2half2_rn(f.x, f.y);
                    w4[j] = *reinterpret_cast<const uint32_t*>(&h);
                }
                qv[i] = x;
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(C::B_QCONV + qb));
            for (int t = sg.t0; t < sg.t1 && ok; ++t, ++g) {
                const int stk = g % C::STK, stv = g % C::STV;
                ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_KFULL + stk), (g / C::STK) & 1, wmisc, p));
                if (!ok) break;
                dec_widen_stage<C>(smem + C::OFF_K + stk * C::KV_BYTES, ct, C::BN);
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::B_KCONV + stk));
                ok = __all_sync(0xffffffffu, wait_bar(bar(C::B_VFULL + stv), (g / C::STV) & 1, wmisc, p));
                if (!ok) break;
                // rows at or past the logical length reach the MMA as zeros (0 * NaN = NaN)
                dec_widen_stage<C>(smem + C::OFF_V + stv * C::KV_BYTES, ct, sg.n - t * C::BN);
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::B_VCONV + stv));
            }
            ++seg_i;
        }
    }

    // ---------------------------------------------------------------- teardown
    // A role ran in one lane of its warp while the other lanes went ahead: the
    // warp reconverges first, so that the CTA barrier below counts every thread
    // (a divergent warp at a CTA barrier can release it early, and TMEM would
    // then be freed while the softmax warps still read it).
    ptx::tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::TM_COLS);
    }
}

}  // namespace gqa
static_assert(sizeof(gqa::DecMisc) <= gqa::DecCfg<8>::MISC_BYTES, "misc block");
