// gqa_fwd2_kernel.cuh -- two-lane sm_100a GQA forward for head dims up to 128.
//
// The CTA keeps two independent online-softmax "lanes" L = 0, 1 in TMEM, each
// with its own S tile (P, as bf16, written back over half of it), its own O
// accumulator and its own softmax warpgroup (4 warps, one per TMEM lane
// quadrant, one packed query row per thread, the whole 128-key row per thread):
//
//   TMEM columns  [0,128) S0/P0   [128,256) S1/P1   [256,256+D) O0   [256+D,256+2D) O1
//
// Two ways to feed the lanes:
//  * split-key (RBQ = 1, at most 128 packed rows: decode, short-q/long-kv):
//    both lanes hold the same 128 packed rows and take alternate key tiles;
//    their (m, l, O) are merged in the segment epilogue.
//  * dual-Q (RBQ = 2, prefill): the lanes hold two consecutive 128-row q-tiles
//    and every K/V tile serves both, which halves the K/V traffic per flop.
// While one warpgroup exponentiates, the other's tile is on the tensor core, so
// softmax latency hides behind MMAs and vice versa.
//
// One thread issues every MMA in this order:
//   split-key: S(g), PV(g-1), S(g+1), PV(g), ...   (S(g) and P(g) in lane g % 2)
//   dual-Q:    S0(j), PV1(j-1), S1(j), PV0(j), ...
// An S MMA into a lane's buffer is always issued after the PV MMA that read the
// lane's previous P from it; the tensor core executes one thread's MMAs in issue
// order, which orders the overwrite after the read.
//
// Warps 0-3: lane 0 softmax; 4-7: lane 1 softmax; 8: Q and K producer (one
// thread); 9: TMEM owner + MMA issuer; 10: split-segment ticket taker; 11: V
// producer.  Each single-thread role has a warp of its own, so no role's spin
// on a barrier delays another's issue.
// Work split, logical-length masking, the sink, split partials and the
// last-arriver merge use the pieces in gqa_common.cuh.
#pragma once
#include "gqa_common.cuh"

namespace gqa {

constexpr int NUM_THREADS2 = 384;  // 12 warps = 3 warpgroups
constexpr int NSOFT2 = 256;        // softmax threads (two warpgroups)
constexpr int kMaxMergeSlots = 64; // pieces a row-block's merge lists in shared memory

template <int D_, int STK_, int STV_, int RBQ_, bool PAGED_ = false>
struct Fwd2Cfg {
    static constexpr int D = D_, BN = 128, STK = STK_, STV = STV_, RBQ = RBQ_;
    static constexpr bool PAGED = PAGED_;  // K/V from a paged cache (chosen at compile time)
    static constexpr bool FP8 = false;     // bf16 K/V
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int NBOX = D / 64;
    static constexpr int Q_BOX = BM * 128;
    static constexpr int Q_TILE = NBOX * Q_BOX;           // one 128-row q-tile
    static constexpr int Q_BYTES = RBQ * Q_TILE;
    static constexpr int KV_BOX = BN * 128;
    static constexpr int KV_BYTES = NBOX * KV_BOX;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + STK * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + STV * KV_BYTES;
    static constexpr int B_QFULL = 0;
    static constexpr int B_QEMPTY = 1;
    static constexpr int B_KFULL = 2;
    static constexpr int B_KEMPTY = B_KFULL + STK;
    static constexpr int B_VFULL = B_KEMPTY + STK;
    static constexpr int B_VEMPTY = B_VFULL + STV;
    static constexpr int B_SFULL = B_VEMPTY + STV;  // [2 lanes]
    static constexpr int B_PFULL = B_SFULL + 2;     // [2 lanes]
    static constexpr int B_ODONE = B_PFULL + 2;     // [2 lanes]
    static constexpr int B_FINAL = B_ODONE + 2;
    static constexpr int B_XSYNC = B_FINAL + 1;
    static constexpr int B_MJOB = B_XSYNC + 1;   // [2] partial rows of split segment j written
    static constexpr int B_MTICK = B_MJOB + 2;   // [2] ticket of split segment j taken
    static constexpr int NBAR = B_MTICK + 2;
    // the control block holds float4-read arrays: 128-byte aligned whatever NBAR is
    static constexpr int OFF_MISC = (OFF_BAR + NBAR * 8 + 127) & ~127;
    static_assert(OFF_MISC % 128 == 0, "control block alignment");
    static constexpr int MISC_BYTES = 2496;
    // the dynamic shared-memory window is required (and checked) to start 1024-aligned
    static constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t TM_COLS = 512;
    __host__ __device__ static constexpr uint32_t tm_s(int L) { return 128u * L; }
    __host__ __device__ static constexpr uint32_t tm_p(int L) { return 128u * L + 64u; }
    __host__ __device__ static constexpr uint32_t tm_o(int L) { return 256u + D * L; }
    static constexpr uint32_t IDESC_S = ptx::umma_idesc_bf16_f32(BM, BN, false, false);
    static constexpr uint32_t IDESC_PV = ptx::umma_idesc_bf16_f32(BM, D, false, true);
};

struct Misc2 {
    uint32_t tmem_base;
    volatile int abort;
    volatile int merge_flag;
    int pad;
    SpanStart span;
    union {
        float st_m[2][BM];    // per-lane row max (log2 domain), by TMEM lane (segment epilogue)
        float mlse[2 * BM];   // merged lse per packed row (in-kernel merge, later)
    };
    float st_l[2][BM];        // per-lane row sum
    int nmerge;               // pieces of the row-block being merged
    int mslot[kMaxMergeSlots];  // their partial slots
    Seg jobs[2];              // this CTA's split segments (its first and last at most)
    int ticket[2];            // 1: this CTA wrote the row-block's last piece and merges it
};

// Part of the softmax exponentials run on the FMA pipe instead of the MUFU unit,
// which computes 16 exp2 per clock per SM: exactly the rate at which the tensor
// pipe consumes a 128 x 128 score tile, so with every exp2 there the two lanes'
// softmaxes are the critical path.  Cody and Waite's range reduction: x = n + f
// with n = round(x) (the 1.5 * 2^23 addition leaves n in the low mantissa bits)
// and f in [-1/2, 1/2]; 2^f by a cubic whose constant term is exactly 1 and whose
// other coefficients minimise the largest relative error on [-1/2, 1/2] (a
// linear program over a fine grid: 1.0e-4, far below the 2^-9 of P's bf16
// rounding); n is added to the exponent field.  x is clamped to -127 first:
// there f = 0, the cubic gives exactly 1.0 and the sum of the fields is +0, so a
// masked score (-inf) still gives an exact 0, and nothing below wraps the field.
// A NaN x gives 0 here, not NaN: rows whose tile maximum is NaN or +inf carry
// a NaN row sum instead (see the softmax).
constexpr float kExp2C1 = 0.693282902f;
constexpr float kExp2C2 = 0.242210969f;
constexpr float kExp2C3 = 0.0550090596f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
__device__ __forceinline__ uint64_t exp2_poly_pair(uint64_t x2) {
    float x0, x1;
    ptx::f2_split(x2, x0, x1);
    const uint64_t xc = ptx::f2(fmaxf(x0, -127.f), fmaxf(x1, -127.f));
    const uint64_t mg = ptx::f2(kRoundMagic, kRoundMagic);
    const uint64_t j = ptx::f2_add(xc, mg);
    const uint64_t f = ptx::f2_sub(xc, ptx::f2_sub(j, mg));
    uint64_t q = ptx::f2_fma(ptx::f2(kExp2C3, kExp2C3), f, ptx::f2(kExp2C2, kExp2C2));
    q = ptx::f2_fma(q, f, ptx::f2(kExp2C1, kExp2C1));
    q = ptx::f2_fma(q, f, ptx::f2(1.f, 1.f));
    float j0, j1, q0, q1;
    ptx::f2_split(j, j0, j1);
    ptx::f2_split(q, q0, q1);
    // the low bits of j are n + 2^22; shifted by 23 only n survives
    const uint32_t r0 = __float_as_uint(q0) + (__float_as_uint(j0) << 23);
    const uint32_t r1 = __float_as_uint(q1) + (__float_as_uint(j1) << 23);
    return ptx::f2(__uint_as_float(r0), __uint_as_float(r1));
}
// Which of the 16 column pairs of each 32-column chunk take the cubic (bit j).
#ifndef GQA_POLY_PAIRS
#define GQA_POLY_PAIRS 0x0u
#endif
constexpr uint32_t kPolyPairs = GQA_POLY_PAIRS;

// Load key tile t of row-block rb (n = its batch's logical length) from K or V
// into one ring stage and arm the stage's full barrier.  Contiguous K/V: one box
// per 64 columns at row rb.kv_row0 + t*BN of the [B*Hkv*Tkv, d] view.  Paged K/V
// ([num_pages, Hkv, page_size, d]): the [num_pages*Hkv*page_size, d] view, one box
// of kv_box_rows (= min(page_size, BN)) rows per page the tile touches, at row
// (page*Hkv + g)*page_size + offset; each lands 8-row aligned in the swizzled
// stage, so the stage holds the same layout as a contiguous tile.
// Pages that start at or past n are not loaded (their rows are masked in S and
// zeroed in V); a page id outside [0, num_pages) is reported and page 0 read.
constexpr int PAGE_BATCH = 4;  // page ids fetched per batch of independent loads

template <class C>
__device__ __forceinline__ void load_kv_tile(const Params& p, const CUtensorMap* tm, uint32_t dst, uint32_t full_bar,
                                             const RB& rb, int t, int n, uint64_t policy) {
    if constexpr (!C::PAGED) {
        ptx::mbar_arrive_expect_tx(full_bar, C::NBOX * p.kv_box_rows * 128);
        const int y = static_cast<int>(rb.kv_row0 + static_cast<long long>(t) * C::BN);
        for (int bx = 0; bx < C::NBOX; ++bx) ptx::tma_load_2d(dst + bx * C::KV_BOX, tm, bx * 64, y, full_bar, policy);
        return;
    }
    const int pr = p.kv_box_rows;
    const int key0 = t * C::BN;
    int nload = 0;
    for (int i = 0; i < C::BN / pr; ++i) nload += (key0 + i * pr < n) ? 1 : 0;
    ptx::mbar_arrive_expect_tx(full_bar, nload * C::NBOX * pr * 128);
    // The page ids are fetched four at a time (independent loads) and the issue
    // loop stays rolled: this code runs beside the unrolled softmax, and fully
    // unrolling it (16 page slots x boxes) measured 2.8x slower for the whole kernel.
    const int sh = 31 - __clz(p.page_size);  // page_size is a power of two
    const int* row_pages = p.page_table + static_cast<long long>(rb.b) * p.max_pages;
#pragma unroll 1
    for (int i0 = 0; i0 < nload; i0 += PAGE_BATCH) {
        int page[PAGE_BATCH];
#pragma unroll
        for (int j = 0; j < PAGE_BATCH; ++j)
            page[j] = (i0 + j < nload) ? __ldg(row_pages + ((key0 + (i0 + j) * pr) >> sh)) : 0;
#pragma unroll
        for (int j = 0; j < PAGE_BATCH; ++j) {
            if (i0 + j >= nload) break;
            int pg = page[j];
            if (pg < 0 || pg >= p.num_pages) {
                atomicCAS(p.err, 0, DEV_ERR_PAGE);
                pg = 0;
            }
            const int key = key0 + (i0 + j) * pr;
            const int y = (pg * p.Hkv + rb.g) * p.page_size + (key & (p.page_size - 1));
#pragma unroll 1
            for (int bx = 0; bx < C::NBOX; ++bx)
                ptx::tma_load_2d(dst + bx * C::KV_BOX + (i0 + j) * pr * 128, tm, bx * 64, y, full_bar, policy);
        }
    }
}

template <class C>
__global__ void __launch_bounds__(NUM_THREADS2, 1)
gqa_fwd2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw;
    const uint32_t sbase = ptx::smem_addr(smem);
    if (sbase & 1023u) {  // the swizzled tiles need a 1024-aligned window
        if (threadIdx.x == 0) atomicCAS(p.err, 0, DEV_ERR_SMEM_ALIGN);
        return;
    }
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
    Misc2* misc = reinterpret_cast<Misc2*>(smem + C::OFF_MISC);
    Misc* wmisc = reinterpret_cast<Misc*>(misc);  // abort flag shared with wait_bar

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const int NC = gridDim.x;

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        ptx::mbar_init(bar(C::B_QFULL), 1);
        ptx::mbar_init(bar(C::B_QEMPTY), 1);
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
            ptx::mbar_init(bar(C::B_PFULL + i), 4);  // one arrival per warp of the lane's warpgroup
            ptx::mbar_init(bar(C::B_ODONE + i), 1);
        }
        ptx::mbar_init(bar(C::B_FINAL), 1);
        ptx::mbar_init(bar(C::B_XSYNC), NSOFT2 / 32);
        for (int j = 0; j < 2; ++j) {
            ptx::mbar_init(bar(C::B_MJOB + j), 1);
            ptx::mbar_init(bar(C::B_MTICK + j), 1);
        }
        misc->abort = 0;
        misc->merge_flag = 0;
        if (p.mode != 0) {
            misc->span.tot = 0;
            misc->span.p0 = misc->span.p1 = 0;
            misc->span.w = misc->span.t = 0;
        }
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tm_q);
        ptx::tma_prefetch_desc(&tm_k);
        ptx::tma_prefetch_desc(&tm_v);
    }
    if (warp == 9) {
        ptx::tmem_alloc(ptx::smem_addr(&misc->tmem_base), C::TM_COLS);
        ptx::tmem_relinquish();
    }
    if (p.mode == 0 && warp == 8) plan_span(p, cta, NC, &misc->span);
    ptx::tc_fence_before();
    __syncwarp();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp >= 8) {
        // 128 x 88 + 256 x 208 = 384 x 168, the registers the block is launched with
        ptx::regs_dec<88>();
        // ------------------------------------------------------------ producers
        if (warp == 8 && lane == 0) {
            // one row-block per KV head (QW == 1): Q serves every tile and K/V stream
            // once; several row-blocks per KV head (prefill): each Q tile is read once
            // and every row-block of the head reads the head's K/V again, so K/V stay
            // in L2 ahead of Q (and of O, written with a streaming hint)
            const uint64_t pol_q = (p.QW == 1) ? ptx::policy_evict_last() : ptx::policy_evict_first();
            const uint64_t pol_kv = (p.QW == 1) ? ptx::policy_evict_first() : ptx::policy_evict_last();
            SegWalker wk;
            wk.init(p, misc->span, cta);
            Seg sg;
            int seg_i = 0;
            uint32_t g = 0;
            bool ok = true;
            uint32_t k_issued[C::STK], q_issued = 0;
            for (int i = 0; i < C::STK; ++i) k_issued[i] = 0;
            while (ok && wk.next(p, sg)) {
                if (sg.t1 <= sg.t0) continue;
                const RB rb = rb_of(p, sg.w);
                ok = wait_bar(bar(C::B_QEMPTY), (seg_i & 1) ^ 1, wmisc, p);
                if (!ok) break;
                // q-tiles of this row-block that exist; the spread layout uses four short boxes
                const int ntile = (rb.rows_valid > BM) ? 2 : 1;
                const int nq = p.spread ? 4 : 1;
                ptx::mbar_arrive_expect_tx(bar(C::B_QFULL), ntile * nq * C::NBOX * p.q_box_rows * 128);
                ++q_issued;
                for (int qt = 0; qt < ntile; ++qt)
                    for (int qq = 0; qq < nq; ++qq)
                        for (int bx = 0; bx < C::NBOX; ++bx)
                            ptx::tma_load_2d(sbase + C::OFF_Q + qt * C::Q_TILE + bx * C::Q_BOX + qq * 32 * 128, &tm_q,
                                             bx * 64, static_cast<int>(rb.q_row0) + qt * BM + qq * p.rq,
                                             bar(C::B_QFULL), pol_q);
                for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                    const int st = g % C::STK;
                    ok = wait_bar(bar(C::B_KEMPTY + st), ((g / C::STK) & 1) ^ 1, wmisc, p);
                    if (!ok) break;
                    ++k_issued[st];
                    load_kv_tile<C>(p, &tm_k, sbase + C::OFF_K + st * C::KV_BYTES, bar(C::B_KFULL + st), rb, t, sg.n, pol_kv);
                }
                ++seg_i;
            }
            for (int i = 0; i < C::STK; ++i) drain_bar(bar(C::B_KFULL + i), k_issued[i], p.timeout_cycles);
            drain_bar(bar(C::B_QFULL), q_issued, p.timeout_cycles);
        } else if (warp == 11 && lane == 0) {
            const uint64_t pol_kv = (p.QW == 1) ? ptx::policy_evict_first() : ptx::policy_evict_last();
            SegWalker wk;
            wk.init(p, misc->span, cta);
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
                    load_kv_tile<C>(p, &tm_v, sbase + C::OFF_V + st * C::KV_BYTES, bar(C::B_VFULL + st), rb, t, sg.n, pol_kv);
                }
            }
            for (int i = 0; i < C::STV; ++i) drain_bar(bar(C::B_VFULL + i), v_issued[i], p.timeout_cycles);
        }
        // ------------------------------------------------------------ MMA issuer
        else if (warp == 9 && lane == 0) {
            SegWalker wk;
            wk.init(p, misc->span, cta);
            Seg sg;
            int seg_i = 0;
            uint32_t g = 0;
            uint32_t n_pv[2] = {0, 0};  // PVs issued per lane (P-full phases consumed)
            bool ok = true;
            // pending split-key PV of tile g-1
            bool have_prev = false;
            int prev_lane = 0, prev_stv = 0;
            bool prev_first = false;
            // pending dual-Q PV of lane 1 for tile j-1
            bool have_b = false, b_first = false;
            int b_stv = 0;

            auto issue_s = [&](int L, uint32_t qbase, uint32_t kbase) {
                const uint32_t d = tmem + C::tm_s(L);
#pragma unroll
                for (int kk = 0; kk < C::D / 16; ++kk) {
                    const uint32_t off = (kk & 3) * 32;
                    const uint64_t ad = ptx::umma_desc_sw128(qbase + (kk >> 2) * C::Q_BOX + off, 16, 1024);
                    const uint64_t bd = ptx::umma_desc_sw128(kbase + (kk >> 2) * C::KV_BOX + off, 16, 1024);
                    ptx::umma_bf16_ss(d, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
                }
                ptx::umma_commit(bar(C::B_SFULL + L));
            };
            // PV of lane L reading V stage st; waits for the lane's P first
            auto issue_pv = [&](int L, int st, bool first, bool wait_v, uint32_t gv) -> bool {
                if (!wait_bar(bar(C::B_PFULL + L), n_pv[L] & 1, wmisc, p)) return false;
                ++n_pv[L];
                if (wait_v && !wait_bar(bar(C::B_VFULL + st), (gv / C::STV) & 1, wmisc, p)) return false;
                ptx::tc_fence_after();
                const uint32_t vbase = sbase + C::OFF_V + st * C::KV_BYTES;
                const uint32_t a = tmem + C::tm_p(L);
                const uint32_t d = tmem + C::tm_o(L);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    const uint64_t bd = ptx::umma_desc_sw128(vbase + kk * 2048, C::KV_BOX, 1024);
                    ptx::umma_bf16_ts(d, a + kk * 8, bd, C::IDESC_PV, (kk > 0 || !first) ? 1u : 0u);
                }
                ptx::umma_commit(bar(C::B_ODONE + L));
                return true;
            };

            while (ok && wk.next(p, sg)) {
                if (sg.t1 <= sg.t0) continue;
                // the previous segment's last PV goes out before this segment's Q is
                // awaited: that segment's epilogue waits for the PV, and the new Q
                // may still be in flight
                if (C::RBQ == 1 && have_prev) {
                    ok = issue_pv(prev_lane, prev_stv, prev_first, true, g - 1);
                    if (!ok) break;
                    ptx::umma_commit(bar(C::B_VEMPTY + prev_stv));
                    have_prev = false;
                }
                if (C::RBQ == 2 && have_b) {
                    ok = issue_pv(1, b_stv, b_first, false, 0);
                    if (!ok) break;
                    ptx::umma_commit(bar(C::B_VEMPTY + b_stv));
                    have_b = false;
                }
                ok = wait_bar(bar(C::B_QFULL), seg_i & 1, wmisc, p);
                if (!ok) break;
                const uint32_t qbase = sbase + C::OFF_Q;
                bool lane_seen[2] = {false, false};
                for (int t = sg.t0; t < sg.t1 && ok; ++t, ++g) {
                    const int stk = g % C::STK;
                    const int stv = g % C::STV;
                    const uint32_t kbase = sbase + C::OFF_K + stk * C::KV_BYTES;
                    // dual-Q: S0 of every tile but a segment's first went out at the end of
                    // the previous iteration, its K stage awaited there
                    if (C::RBQ == 1 || t == sg.t0) {
                        ok = wait_bar(bar(C::B_KFULL + stk), (g / C::STK) & 1, wmisc, p);
                        if (!ok) break;
                        ptx::tc_fence_after();
                    }
                    if (C::RBQ == 1) {
                        const int L = g & 1;
                        issue_s(L, qbase, kbase);
                        ptx::umma_commit(bar(C::B_KEMPTY + stk));
                        if (t == sg.t1 - 1) ptx::umma_commit(bar(C::B_QEMPTY));
                        if (have_prev) {
                            ok = issue_pv(prev_lane, prev_stv, prev_first, true, g - 1);
                            if (!ok) break;
                            ptx::umma_commit(bar(C::B_VEMPTY + prev_stv));
                        }
                        have_prev = true;
                        prev_lane = L;
                        prev_stv = stv;
                        prev_first = !lane_seen[L];
                        lane_seen[L] = true;
                    } else {
                        // A wait in this thread stalls the tensor pipe for about 130 cycles
                        // even on a completed barrier, so lane 0's chain (P0 -> PV0 -> next
                        // S0 -> softmax) keeps one wait, on P0: V(t) and K(t+1) are awaited
                        // while S1(t) executes.
                        if (t == sg.t0) issue_s(0, qbase, kbase);
                        if (have_b) {
                            ok = issue_pv(1, b_stv, b_first, false, 0);
                            if (!ok) break;
                            ptx::umma_commit(bar(C::B_VEMPTY + b_stv));
                        }
                        issue_s(1, qbase + C::Q_TILE, kbase);
                        ptx::umma_commit(bar(C::B_KEMPTY + stk));
                        if (t == sg.t1 - 1) ptx::umma_commit(bar(C::B_QEMPTY));
                        ok = wait_bar(bar(C::B_VFULL + stv), (g / C::STV) & 1, wmisc, p);
                        if (!ok) break;
                        const bool more = t + 1 < sg.t1;
                        const int stk1 = (g + 1) % C::STK;
                        if (more) {
                            ok = wait_bar(bar(C::B_KFULL + stk1), ((g + 1) / C::STK) & 1, wmisc, p);
                            if (!ok) break;
                        }
                        ok = issue_pv(0, stv, t == sg.t0, false, g);
                        if (!ok) break;
                        if (more) issue_s(0, qbase, sbase + C::OFF_K + stk1 * C::KV_BYTES);
                        have_b = true;
                        b_first = (t == sg.t0);
                        b_stv = stv;
                    }
                }
                ++seg_i;
            }
            if (ok && C::RBQ == 1 && have_prev) {
                ok = issue_pv(prev_lane, prev_stv, prev_first, true, g - 1);
                if (ok) ptx::umma_commit(bar(C::B_VEMPTY + prev_stv));
            }
            if (ok && C::RBQ == 2 && have_b) {
                ok = issue_pv(1, b_stv, b_first, false, 0);
                if (ok) ptx::umma_commit(bar(C::B_VEMPTY + b_stv));
            }
            ptx::umma_commit(bar(C::B_FINAL));
            drain_bar(bar(C::B_FINAL), 1, p.timeout_cycles);
        }
        // ------------------------------------------------------------ ticket taker
        // For each split segment: once the softmax warps have written its partial
        // rows, publish them (release fence) and count this CTA's piece of the
        // row-block; the CTA whose count completes it merges the pieces.  The
        // softmax warps do not wait for this until their last segment is done.
        else if (warp == 10 && lane == 0) {
            SegWalker wk;
            wk.init(p, misc->span, cta);
            Seg sg;
            int j = 0;
            const long long tot = misc->span.tot;
            while (j < 2 && wk.next(p, sg)) {
                if (sg.kind != 1) continue;
                if (!wait_bar(bar(C::B_MJOB + j), 0, wmisc, p)) break;
                const int c_first = cta_of(sg.pw, tot, NC);
                const int c_last = cta_of(sg.pw + sg.ntiles - 1, tot, NC);
                int ncontrib = 0;
                for (int cc = c_first; cc <= c_last; ++cc) ncontrib += span_begin(cc, tot, NC) < span_begin(cc + 1, tot, NC);
                __threadfence();
                const int old = atomicAdd(p.counters + sg.w, 1);
                misc->ticket[j] = (old == ncontrib - 1);
                ptx::mbar_arrive(bar(C::B_MTICK + j));
                ++j;
            }
        }
    }
    // ---------------------------------------------------------------- softmax lanes
    else {
        ptx::regs_inc<208>();
        const int L = warp >> 2;               // lane (warpgroup)
        const int quad = warp & 3;             // TMEM lane quadrant
        const int lrow = quad * 32 + lane;     // TMEM lane = row of the MMA tile
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const int stid = threadIdx.x;          // 0..255
        const int wtid = threadIdx.x & 127;    // index inside the lane's warpgroup
        uint32_t xph = 0;
        auto xsync = [&]() -> bool {           // both softmax warpgroups, bounded
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(C::B_XSYNC));
            const bool r = wait_bar(bar(C::B_XSYNC), xph & 1, wmisc, p);
            ++xph;
            ptx::tc_fence_after();
            return __all_sync(0xffffffffu, r);
        };
        SegWalker wk;
        wk.init(p, misc->span, cta);
        Seg sg;
        uint32_t g = 0;
        uint32_t cnt = 0;  // tiles this lane has processed (barrier phases)
        bool ok = true;
        int njob = 0;      // split segments handed to the ticket taker

        while (ok && wk.next(p, sg)) {
            const RB rb = rb_of(p, sg.w);
            // rows this lane's thread owns: dual-Q lane L takes the L-th q-tile
            const int tile_row0 = (C::RBQ == 2) ? L * BM : 0;
            const int rows_here = rb.rows_valid - tile_row0;  // rows of this lane's q-tile (may be <= 0)
            int rloc;
            bool valid, active;
            if (p.spread) {
                rloc = quad * p.rq + lane;
                valid = lane < p.rq && rloc < rows_here;
                active = quad * p.rq < rows_here;
            } else {
                rloc = lrow;
                valid = lrow < rows_here;
                active = quad * 32 < rows_here;
            }
            const int rrb = tile_row0 + rloc;        // row inside the row-block
            const int rp = rb.qt * BM + rrb;         // packed row inside the unit
            const int hl = valid ? rp / p.Tq : 0;
            const int i = valid ? rp % p.Tq : 0;
            int limit = p.causal ? (sg.n - p.Tq + i) : (sg.n - 1);
            if (limit > sg.n - 1) limit = sg.n - 1;
            if (!valid) limit = -1;
            const int h = rb.g * p.G + hl;

            float m_ref = -INFINITY;
            float l_sum = 0.f;
            int mine = 0;  // tiles of this segment processed by this lane

            for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                if (C::RBQ == 1 && static_cast<int>(g & 1) != L) continue;
                ok = wait_bar(bar(C::B_SFULL + L), cnt & 1, wmisc, p);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ptx::tc_fence_after();
                const bool first = (mine == 0);
                float alpha = 1.f;
                if (active) {
                    float s[C::BN];
                    const uint32_t ts = tmem + lane_off + C::tm_s(L);
#pragma unroll
                    for (int c = 0; c < C::BN / 32; ++c) {
                        uint32_t r[32];
                        ptx::tmem_ld32(ts + c * 32, r);
#pragma unroll
                        for (int j = 0; j < 32; ++j) s[c * 32 + j] = __uint_as_float(r[j]);
                    }
                    ptx::tmem_wait_ld();
                    // mask by selection (never by adding -inf: NaN + -inf stays NaN)
                    const int lim = limit - t * C::BN;
                    if (!__all_sync(0xffffffffu, lim >= C::BN - 1)) {
#pragma unroll
                        for (int c = 0; c < C::BN; ++c) s[c] = (c <= lim) ? s[c] : -INFINITY;
                    }
                    // the tile maximum; NaN if any visible score is NaN
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < C::BN; c += 8) {
                        m4[0] = ptx::max3_nan(m4[0], s[c], s[c + 1]);
                        m4[1] = ptx::max3_nan(m4[1], s[c + 2], s[c + 3]);
                        m4[2] = ptx::max3_nan(m4[2], s[c + 4], s[c + 5]);
                        m4[3] = ptx::max3_nan(m4[3], s[c + 6], s[c + 7]);
                    }
                    const float mt = ptx::max3_nan(m4[0], m4[1], ptx::max3_nan(m4[2], m4[3], m4[3])) * p.scale_log2;
                    if (first) {
                        m_ref = mt;
                    } else if (mt > m_ref + RESCALE_THRESHOLD) {
                        alpha = ptx::ex2(m_ref - mt);
                        m_ref = mt;
                    }
                    // P = 2^(s*scale*log2e - m) as bf16 over the lane's S columns [64, 128)
                    const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
                    const uint32_t tp = tmem + lane_off + C::tm_p(L);
                    const uint64_t sl2 = ptx::f2(p.scale_log2, p.scale_log2);
                    const uint64_t nm2 = ptx::f2(neg_m, neg_m);
                    uint64_t acc[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) acc[a] = ptx::f2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < C::BN / 32; ++c) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const uint64_t x2 = ptx::f2_fma(ptx::f2(s[c * 32 + 2 * j], s[c * 32 + 2 * j + 1]), sl2, nm2);
                            uint64_t e2;
                            if ((kPolyPairs >> j) & 1u) {
                                e2 = exp2_poly_pair(x2);
                            } else {
                                float x0, x1;
                                ptx::f2_split(x2, x0, x1);
                                e2 = ptx::f2(ptx::ex2(x0), ptx::ex2(x1));
                            }
                            acc[j & 3] = ptx::f2_add(acc[j & 3], e2);
                            float e0, e1;
                            ptx::f2_split(e2, e0, e1);
                            pk[j] = pack_bf16x2(e0, e1);
                        }
                        ptx::tmem_st16(tp + c * 16, pk);
                    }
                    float a0, a1;
                    ptx::f2_split(ptx::f2_add(ptx::f2_add(acc[0], acc[1]), ptx::f2_add(acc[2], acc[3])), a0, a1);
                    l_sum = l_sum * alpha + (a0 + a1);
                    // a NaN or +inf maximum: the cubic turned NaN scores into 0, so mark the row
                    if (mt != mt || mt == INFINITY) l_sum = __int_as_float(0x7fffffff);
                }
                // lazy rescale of the lane's O: only when a row's max grew by more than 2^8
                if (!first && __any_sync(0xffffffffu, alpha != 1.f)) {
                    bool okw = wait_bar(bar(C::B_ODONE + L), (cnt - 1) & 1, wmisc, p);
                    okw = __all_sync(0xffffffffu, okw);
                    if (!okw) {
                        ok = false;
                    } else {
                        ptx::tc_fence_after();
                        const uint32_t to = tmem + lane_off + C::tm_o(L);
#pragma unroll 1
                        for (int c = 0; c < C::D / 32; ++c) {
                            uint32_t r[32];
                            ptx::tmem_ld32(to + c * 32, r);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
                            ptx::tmem_st32(to + c * 32, r);
                        }
                    }
                }
                if (active) ptx::tmem_wait_st();
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                // padded key rows of the V tile reach the MMA as zeros (0 * NaN = NaN)
                if ((t + 1) * C::BN > sg.n) {
                    const int st = g % C::STV;
                    ok = wait_bar(bar(C::B_VFULL + st), (g / C::STV) & 1, wmisc, p);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    int z0 = sg.n - t * C::BN;
                    z0 = z0 < 0 ? 0 : z0;
                    uint8_t* vt = smem + C::OFF_V + st * C::KV_BYTES;
                    const int chunks = (C::BN - z0) * C::NBOX * 8;
                    for (int q = wtid; q < chunks; q += 128) {
                        const int r = z0 + q / (C::NBOX * 8);
                        const int rem = q % (C::NBOX * 8);
                        *reinterpret_cast<uint4*>(vt + (rem >> 3) * C::KV_BOX + r * 128 + (rem & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::B_PFULL + L));
                ++cnt;
                ++mine;
            }
            if (!ok) break;

            // ------------------------------------------------ segment epilogue
            if (mine > 0) {
                ok = wait_bar(bar(C::B_ODONE + L), (cnt - 1) & 1, wmisc, p);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ptx::tc_fence_after();
            }
            const long long fr = rb.q_row0 + rrb;  // flat row (b*Hq + h)*Tq + i when valid
            // final weights of the lane accumulators for this thread's row:
            //   out = w0 * O0 + w1 * O1   (split-key: both lanes, same rows; dual-Q: own lane only)
            float w_own = 0.f, w_oth = 0.f, lse_v = -INFINITY;
            const bool direct = (sg.kind == 0);
            if (C::RBQ == 1) {
                misc->st_m[L][lrow] = (mine > 0) ? m_ref : -INFINITY;
                misc->st_l[L][lrow] = (mine > 0) ? l_sum : 0.f;
                if (!xsync()) { ok = false; break; }
                const float mo = misc->st_m[L ^ 1][lrow], lo = misc->st_l[L ^ 1][lrow];
                const float mm = (mine > 0) ? m_ref : -INFINITY, ll = (mine > 0) ? l_sum : 0.f;
                const float sk = (direct && p.sink != nullptr && valid) ? __ldg(p.sink + h) * LOG2E : -INFINITY;
                const float M = fmax_nan(fmax_nan(mm, mo), sk);
                if (M != -INFINITY) {
                    const float a = pos_or_nan(ll) ? ptx::ex2(mm - M) : 0.f;
                    const float b = pos_or_nan(lo) ? ptx::ex2(mo - M) : 0.f;
                    const float lt = ll * a + lo * b + ((sk != -INFINITY) ? ptx::ex2(sk - M) : 0.f);
                    if (pos_or_nan(lt)) {
                        w_own = a / lt;
                        w_oth = b / lt;
                        lse_v = (M + __log2f(lt)) * LN2;
                    }
                }
            } else {
                const float sk = (direct && p.sink != nullptr && valid) ? __ldg(p.sink + h) * LOG2E : -INFINITY;
                const float M = fmax_nan(m_ref, sk);
                if (M != -INFINITY) {
                    const float a = pos_or_nan(l_sum) ? ptx::ex2(m_ref - M) : 0.f;
                    const float lt = l_sum * a + ((sk != -INFINITY) ? ptx::ex2(sk - M) : 0.f);
                    if (pos_or_nan(lt)) {
                        w_own = a / lt;
                        lse_v = (M + __log2f(lt)) * LN2;
                    }
                }
            }
            // columns this thread writes: split-key halves D between the lanes
            constexpr int SPLIT_COLS = C::D / 2;
            const int c0 = (C::RBQ == 1) ? L * SPLIT_COLS : 0;
            const int ncol = (C::RBQ == 1) ? SPLIT_COLS : C::D;
            const uint32_t to_own = tmem + lane_off + C::tm_o(L) + c0;
            const uint32_t to_oth = tmem + lane_off + C::tm_o(L ^ 1) + c0;
            float* pdst = nullptr;
            float* pdl = nullptr;
            if (sg.kind == 1) {
                pdst = p.part_o + (static_cast<long long>(sg.slot) * (BM * C::RBQ) + rrb) * C::D + c0;
                pdl = p.part_lse + static_cast<long long>(sg.slot) * (BM * C::RBQ) + rrb;
            } else if (sg.kind == 2) {
                pdst = p.part_o + (fr * p.num_splits + sg.slot) * C::D + c0;
                pdl = p.part_lse + fr * p.num_splits + sg.slot;
            }
            if (active) {
#pragma unroll 1
                for (int c = 0; c < ncol / 32; ++c) {
                    uint32_t ro[32], rx[32];
                    ptx::tmem_ld32(to_own + c * 32, ro);
                    if (C::RBQ == 1) ptx::tmem_ld32(to_oth + c * 32, rx);
                    ptx::tmem_wait_ld();
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        float x = (w_own != 0.f) ? __uint_as_float(ro[j]) * w_own : 0.f;
                        if (C::RBQ == 1 && w_oth != 0.f) x += __uint_as_float(rx[j]) * w_oth;
                        v[j] = x;
                    }
                    if (valid) {
                        if (direct) {
                            uint4* d4 = reinterpret_cast<uint4*>(p.out + fr * C::D + c0 + c * 32);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                __stcs(d4 + j, make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                                          pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                                          pack_bf16x2(v[8 * j + 6], v[8 * j + 7])));
                        } else {
                            float4* d4 = reinterpret_cast<float4*>(pdst + c * 32);
#pragma unroll
                            for (int j = 0; j < 8; ++j) __stcg(d4 + j, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
                        }
                    }
                }
            }
            const bool writes_lse = valid && (C::RBQ == 2 || L == 0);
            if (writes_lse) {
                if (direct) {
                    if (p.lse != nullptr) p.lse[fr] = lse_v;
                } else {
                    __stcg(pdl, lse_v);
                }
            }
            // both lanes' O reads are done before the next segment's first PVs
            // overwrite them; a split segment's partial rows are written
            if (!xsync()) { ok = false; break; }
            if (sg.kind == 1 && njob < 2) {
                if (stid == 0) {
                    misc->jobs[njob] = sg;
                    ptx::mbar_arrive(bar(C::B_MJOB + njob));
                }
                ++njob;
            }
            ptx::tc_fence_before();
        }
        // merges of the row-blocks whose last piece this CTA wrote
        for (int j = 0; ok && j < njob; ++j) {
            ok = wait_bar(bar(C::B_MTICK + j), 0, wmisc, p);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (!misc->ticket[j]) continue;
            __threadfence();
            const Seg sg = misc->jobs[j];
            const RB rb = rb_of(p, sg.w);
            const long long tot = misc->span.tot;
            const int c_first = cta_of(sg.pw, tot, NC);
            const int c_last = cta_of(sg.pw + sg.ntiles - 1, tot, NC);
            {
                const bool c0_first = span_begin(c_first, tot, NC) == sg.pw;
                const long long RW = BM * C::RBQ;
                // slots of the CTAs that hold a piece of this row-block, compacted
                if (warp == 0) {
                    int nm = 0;
                    for (int base = c_first; base <= c_last; base += 32) {
                        const int cc = base + lane;
                        const bool has = cc <= c_last && span_begin(cc, tot, NC) < span_begin(cc + 1, tot, NC);
                        const unsigned m = __ballot_sync(0xffffffffu, has);
                        const int k = nm + __popc(m & ((1u << lane) - 1u));
                        if (has && k < kMaxMergeSlots) misc->mslot[k] = merge_slot(cc, c_first, c0_first);
                        nm += __popc(m);
                    }
                    if (lane == 0) misc->nmerge = nm;
                }
                if (!xsync()) { ok = false; break; }
                const int nm = misc->nmerge;
                if (nm <= kMaxMergeSlots) {
                    // lse of each merged row: all partial lse loads issued together
                    for (int r = stid; r < rb.rows_valid; r += NSOFT2) {
                        const int hr = rb.g * p.G + (rb.qt * BM + r) / p.Tq;
                        const float sk = (p.sink != nullptr) ? __ldg(p.sink + hr) : -INFINITY;
                        float Lx = sk;
                        float lv[8];
                        for (int k0 = 0; k0 < nm; k0 += 8) {
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                lv[j] = (k0 + j < nm) ? __ldcg(p.part_lse + misc->mslot[k0 + j] * RW + r) : -INFINITY;
#pragma unroll
                            for (int j = 0; j < 8; ++j) Lx = fmax_nan(Lx, lv[j]);
                        }
                        float lt = -INFINITY;
                        if (Lx != -INFINITY) {
                            float z = (sk != -INFINITY) ? __expf(sk - Lx) : 0.f;
                            if (nm <= 8) {
#pragma unroll
                                for (int j = 0; j < 8; ++j) z += __expf(lv[j] - Lx);
                            } else {
                                for (int k = 0; k < nm; ++k) z += __expf(__ldcg(p.part_lse + misc->mslot[k] * RW + r) - Lx);
                            }
                            lt = Lx + __logf(z);
                        }
                        misc->mlse[r] = lt;
                        if (p.lse != nullptr) p.lse[rb.q_row0 + r] = lt;
                    }
                    if (!xsync()) { ok = false; break; }
                    // O rows: weight exp(lse_k - lse) per piece; four pieces' loads in flight at once
                    constexpr int C8 = C::D / 8;
                    for (int it = stid; it < rb.rows_valid * C8; it += NSOFT2) {
                        const int r = it / C8, c8 = it % C8;
                        const float lt = misc->mlse[r];
                        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        if (lt != -INFINITY) {
                            for (int k0 = 0; k0 < nm; k0 += 4) {
                                float lw[4];
                                float4 xa[4], xb[4];
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    if (k0 + j < nm) {
                                        const long long sl = misc->mslot[k0 + j];
                                        const float4* src = reinterpret_cast<const float4*>(p.part_o + (sl * RW + r) * C::D + 8 * c8);
                                        lw[j] = __ldcg(p.part_lse + sl * RW + r);
                                        xa[j] = __ldcg(src);
                                        xb[j] = __ldcg(src + 1);
                                    } else {
                                        lw[j] = -INFINITY;
                                        xa[j] = xb[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                                    }
                                }
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const float wgt = __expf(lw[j] - lt);
                                    acc[0] += wgt * xa[j].x; acc[1] += wgt * xa[j].y; acc[2] += wgt * xa[j].z; acc[3] += wgt * xa[j].w;
                                    acc[4] += wgt * xb[j].x; acc[5] += wgt * xb[j].y; acc[6] += wgt * xb[j].z; acc[7] += wgt * xb[j].w;
                                }
                            }
                        }
                        *reinterpret_cast<uint4*>(p.out + (rb.q_row0 + r) * C::D + 8 * c8) =
                            make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                       pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
                    }
                } else {
                    // more pieces than the slot list holds: walk the CTAs again
                    for (int r = stid; r < rb.rows_valid; r += NSOFT2) {
                        const int hr = rb.g * p.G + (rb.qt * BM + r) / p.Tq;
                        float Lx = (p.sink != nullptr) ? __ldg(p.sink + hr) : -INFINITY;
                        for (int cc = c_first; cc <= c_last; ++cc) {
                            if (!(span_begin(cc, tot, NC) < span_begin(cc + 1, tot, NC))) continue;
                            Lx = fmax_nan(Lx, __ldcg(p.part_lse + merge_slot(cc, c_first, c0_first) * RW + r));
                        }
                        float lt = -INFINITY;
                        if (Lx != -INFINITY) {
                            float z = (p.sink != nullptr) ? __expf(__ldg(p.sink + hr) - Lx) : 0.f;
                            for (int cc = c_first; cc <= c_last; ++cc) {
                                if (!(span_begin(cc, tot, NC) < span_begin(cc + 1, tot, NC))) continue;
                                z += __expf(__ldcg(p.part_lse + merge_slot(cc, c_first, c0_first) * RW + r) - Lx);
                            }
                            lt = Lx + __logf(z);
                        }
                        misc->mlse[r] = lt;
                        if (p.lse != nullptr) p.lse[rb.q_row0 + r] = lt;
                    }
                    if (!xsync()) { ok = false; break; }
                    constexpr int C8 = C::D / 8;
                    for (int it = stid; it < rb.rows_valid * C8; it += NSOFT2) {
                        const int r = it / C8, c8 = it % C8;
                        const float lt = misc->mlse[r];
                        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        if (lt != -INFINITY) {
                            for (int cc = c_first; cc <= c_last; ++cc) {
                                if (!(span_begin(cc, tot, NC) < span_begin(cc + 1, tot, NC))) continue;
                                const long long sl = merge_slot(cc, c_first, c0_first);
                                const float wgt = __expf(__ldcg(p.part_lse + sl * RW + r) - lt);
                                const float4* src = reinterpret_cast<const float4*>(p.part_o + (sl * RW + r) * C::D + 8 * c8);
                                const float4 xa = __ldcg(src), xb = __ldcg(src + 1);
                                acc[0] += wgt * xa.x; acc[1] += wgt * xa.y; acc[2] += wgt * xa.z; acc[3] += wgt * xa.w;
                                acc[4] += wgt * xb.x; acc[5] += wgt * xb.y; acc[6] += wgt * xb.z; acc[7] += wgt * xb.w;
                            }
                        }
                        *reinterpret_cast<uint4*>(p.out + (rb.q_row0 + r) * C::D + 8 * c8) =
                            make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                       pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
                    }
                }
                if (stid == 0) p.counters[sg.w] = 0;
            }
            if (!xsync()) { ok = false; break; }
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
    if (warp == 9) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::TM_COLS);
    }
}

}  // namespace gqa

static_assert(sizeof(gqa::Misc2) <= 2496, "misc block");
