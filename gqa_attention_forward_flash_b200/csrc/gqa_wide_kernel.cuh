// gqa_wide_kernel.cuh -- sm_100a GQA forward for the wide head dims 256 and 512.
//
// A 128-row tile of packed query rows (the G query heads of one KV head times
// their Tq rows; AstrAI commit log, head-packing commit) against 128-key tiles:
//
//   S = Q K^T   [128 rows x 128 keys] fp32 in TMEM, K-major operands from shared memory
//   O += P V    [128 rows x 256 columns] fp32 in TMEM, P (bf16) from TMEM
//
// With d = 512 a 128 x 512 fp32 O would fill all 512 TMEM columns, so O's columns
// are split over two CTAs (DSPLIT = 2) that walk the same key tiles: each
// computes the full S and keeps 256 columns of O.  The two CTAs of a pair read
// the same K rows at about the same time, so HBM sees each K byte once (the
// second read hits L2); each reads only its own half of V.
//
// Shared memory: the whole Q tile stays resident for the segment (128 KB at
// d = 512); K and V stream through one ring of 16 KB chunks (128 keys x 64
// columns, 128-byte swizzle), in exactly the order the MMA thread consumes
// them: K(g) chunks for S(g), V(g-1) chunks for PV(g-1).  A 128-key S is then
// d/16 MMAs of N = 128 whatever the head dim (a whole K tile would not fit
// beside Q).
//
//   TMEM columns  [0, 256) O   [256, 384) S0 / P0   [384, 512) S1 / P1
//   (P(g), bf16, is written over the upper half of S(g)'s columns)
//
// MMA order (one thread): S(g), PV(g-1), S(g+1), PV(g), ...; at a segment
// switch the previous segment's last PV goes first.  S(g+1) runs on the tensor
// core while the softmax warps work on S(g).
//
// Split row-blocks are merged inside this kernel (NEXT-1 of the split-KV path):
// every CTA that wrote a piece of a split row-block waits, after its own span,
// until all pieces are published and then merges its share of the rows; so a
// row-block cut into k pieces is merged by k CTAs at once (AstrAI commit log:
// the in-kernel fold after an atomic count with fences; kernbench2 benches
// commit log: the associative (m, l, O) merge).  The waits need every CTA of
// the grid resident at once: the grid is at most one CTA per SM and the launch
// is cooperative.
//
// Warps: 0 ring producer (K/V chunks); 1 Q producer; 2 TMEM owner + MMA issuer;
// 3 publisher of split pieces; 4-7 softmax / epilogue / merge (warp 4+q reads
// TMEM lane quadrant q, one packed row per thread).
#pragma once
#include "gqa_common.cuh"

namespace gqa {

constexpr int NUM_THREADS_W = 256;
constexpr int NSOFT_W = 128;
constexpr int kWideSlotCap = 160;    // pieces whose slots the merge lists in shared memory
constexpr int kWideStageMax = 64;    // pieces the merge stages in shared memory at once (more: read in place)

struct WideMisc {
    uint32_t tmem_base;  // the first four fields match Misc (bounded waits read abort)
    volatile int abort;
    volatile int merge_flag;
    int pad;
    SpanStart span;
    Seg jobs[2];                  // this CTA's split segments (its first and last at most)
    int nslot;
    int mslot[kWideSlotCap];      // partial slots of the pieces being merged
    float mlse[BM];               // merged lse per row (merge of many pieces, read in place)
};

template <int D_, int DSPLIT_>
struct WideCfg {
    static constexpr int D = D_, DSPLIT = DSPLIT_, BN = 128;
    static constexpr int DO = D / DSPLIT;  // O columns held by one CTA
    static constexpr bool FP8 = false;     // bf16 K/V
    static_assert((D == 256 && DSPLIT == 1) || (D == 512 && DSPLIT == 2), "head dim");
    static_assert(DO == 256, "O takes 256 TMEM columns");
    static constexpr int NBOX = D / 64;   // K chunks per tile (and Q boxes)
    static constexpr int VCH = DO / 64;   // V chunks per tile (this CTA's columns)
    static constexpr int CH = NBOX + VCH; // ring chunks per tile
    static constexpr int CHUNK = BN * 128;
    static constexpr int Q_BOX = BM * 128;
    static constexpr int Q_BYTES = NBOX * Q_BOX;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_RING = Q_BYTES;
    static constexpr int MISC_BYTES = (static_cast<int>(sizeof(WideMisc)) + 15) & ~15;
    static constexpr int NSLOT = (232448 - Q_BYTES - MISC_BYTES - 40 * 8) / CHUNK;  // 6 at d = 512, 10 at 256
    static constexpr int OFF_BAR = OFF_RING + NSLOT * CHUNK;
    static constexpr int B_QFULL = 0;
    static constexpr int B_QEMPTY = 1;
    static constexpr int B_RFULL = 2;                   // [NSLOT]
    static constexpr int B_REMPTY = B_RFULL + NSLOT;    // [NSLOT]
    static constexpr int B_SFULL = B_REMPTY + NSLOT;    // [2] S(g) in TMEM
    static constexpr int B_PFULL = B_SFULL + 2;         // [2] P(g) in TMEM (one arrival per softmax warp)
    static constexpr int B_ODONE = B_PFULL + 2;         // [2] PV(g) completed
    static constexpr int B_OFREE = B_ODONE + 2;         // a segment's epilogue has read O
    static constexpr int B_FINAL = B_OFREE + 1;
    static constexpr int B_XSYNC = B_FINAL + 1;
    static constexpr int B_MJOB = B_XSYNC + 1;          // [2] partial rows of split segment j written
    static constexpr int B_MERGE = B_MJOB + 2;          // merge: the pieces' staged partials have landed
    static constexpr int NBAR = B_MERGE + 1;
    static_assert(NBAR <= 40, "barrier block");
    static constexpr int OFF_MISC = OFF_BAR + 40 * 8;
    static_assert(OFF_MISC % 16 == 0, "control block alignment");
    static constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t TM_COLS = 512;
    static constexpr uint32_t TM_O = 0;
    static constexpr uint32_t TM_S = 256;  // + 128 * buffer
    static constexpr uint32_t IDESC_S = ptx::umma_idesc_bf16_f32(BM, BN, false, false);
    static constexpr uint32_t IDESC_PV = ptx::umma_idesc_bf16_f32(BM, 64, false, true);
    // stream-K partial slots: [slot][GJ column groups of four][BM rows] float4, so a
    // warp's 32 rows of one column group are 512 contiguous bytes, and one merging
    // CTA's column groups of one piece are one contiguous block
    static constexpr int GJ = DO / 4;
    // merge staging in the (then idle) Q + ring area: the pieces' lse rows, then their O blocks
    static constexpr int STAGE_LSE = 0;
    static constexpr int STAGE_O = kWideStageMax * BM * 4;
    static constexpr int STAGE_END = OFF_BAR;
    static_assert(STAGE_END - STAGE_O >= kWideStageMax * BM * 16, "one column group of every staged piece fits");
    // first ring chunk of V(g) when tile g is the last tile of its segment: the
    // chunk sequence is K(0), then per tile g >= 1 [K(g), V(g-1)] or, where g
    // starts a segment, [V(g-1), K(g)], and V(last) at the end
    __host__ __device__ static constexpr uint32_t v_seq_last_of_segment(uint32_t g) { return NBOX + g * CH; }
};

// Counters of a split row-block w, O part ho: [0] pieces published, [1] pieces merged
__device__ __forceinline__ int* wide_counters(const Params& p, int w, int ho, int dsplit) {
    return p.counters + 2ll * (static_cast<long long>(w) * dsplit + ho);
}

__device__ __forceinline__ int ld_acquire(const int* a) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
    return v;
}

template <class C>
__global__ void __launch_bounds__(NUM_THREADS_W, 1)
gqa_wide_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
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
    WideMisc* misc = reinterpret_cast<WideMisc*>(smem + C::OFF_MISC);
    Misc* wmisc = reinterpret_cast<Misc*>(misc);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // CTAs come in groups of DSPLIT that walk the same work; ho picks the O columns
    const int ho = static_cast<int>(blockIdx.x) % C::DSPLIT;
    const int cta = static_cast<int>(blockIdx.x) / C::DSPLIT;
    const int NC = static_cast<int>(gridDim.x) / C::DSPLIT;

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        ptx::mbar_init(bar(C::B_QFULL), 1);
        ptx::mbar_init(bar(C::B_QEMPTY), 1);
        for (int i = 0; i < C::NSLOT; ++i) {
            ptx::mbar_init(bar(C::B_RFULL + i), 1);
            ptx::mbar_init(bar(C::B_REMPTY + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(C::B_SFULL + i), 1);
            ptx::mbar_init(bar(C::B_PFULL + i), 4);
            ptx::mbar_init(bar(C::B_ODONE + i), 1);
            ptx::mbar_init(bar(C::B_MJOB + i), 1);
        }
        ptx::mbar_init(bar(C::B_OFREE), 4);
        ptx::mbar_init(bar(C::B_FINAL), 1);
        ptx::mbar_init(bar(C::B_XSYNC), 4);
        ptx::mbar_init(bar(C::B_MERGE), 1);
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
    if (warp == 2) {
        ptx::tmem_alloc(ptx::smem_addr(&misc->tmem_base), C::TM_COLS);
        ptx::tmem_relinquish();
    }
    if (p.mode == 0 && warp == 0) plan_span(p, cta, NC, &misc->span);
    ptx::tc_fence_before();
    __syncwarp();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp < 4) {
        // ------------------------------------------------------------ ring producer
        if (warp == 0 && lane == 0) {
            // K rows are read by both CTAs of a pair: normal priority; V once: evict first
            const uint64_t pol_k = (p.QT == 1 && C::DSPLIT == 1) ? ptx::policy_evict_first() : ptx::policy_evict_normal();
            const uint64_t pol_v = (p.QT == 1) ? ptx::policy_evict_first() : ptx::policy_evict_normal();
            SegWalker wk;
            wk.init(p, misc->span, cta);
            Seg sg;
            uint32_t seq = 0;
            bool ok = true;
            uint32_t issued[C::NSLOT];
            for (int i = 0; i < C::NSLOT; ++i) issued[i] = 0;
            auto put = [&](const CUtensorMap* tm, int x, int y, uint64_t pol) -> bool {
                const int s = static_cast<int>(seq % C::NSLOT);
                if (!wait_bar(bar(C::B_REMPTY + s), ((seq / C::NSLOT) & 1) ^ 1, wmisc, p)) return false;
                ptx::mbar_arrive_expect_tx(bar(C::B_RFULL + s), p.kv_box_rows * 128);
                ++issued[s];
                ptx::tma_load_2d(sbase + C::OFF_RING + s * C::CHUNK, tm, x, y, bar(C::B_RFULL + s), pol);
                ++seq;
                return true;
            };
            auto put_k = [&](long long kv_row0, int t) -> bool {
                const int y = static_cast<int>(kv_row0 + static_cast<long long>(t) * C::BN);
                for (int c = 0; c < C::NBOX; ++c)
                    if (!put(&tm_k, c * 64, y, pol_k)) return false;
                return true;
            };
            auto put_v = [&](long long kv_row0, int t) -> bool {
                const int y = static_cast<int>(kv_row0 + static_cast<long long>(t) * C::BN);
                for (int c = 0; c < C::VCH; ++c)
                    if (!put(&tm_v, ho * C::DO + c * 64, y, pol_v)) return false;
                return true;
            };
            bool have_prev = false;
            long long prev_row0 = 0;
            int prev_t = 0;
            while (ok && wk.next(p, sg)) {
                if (sg.t1 <= sg.t0) continue;
                const RB rb = rb_of(p, sg.w);
                for (int t = sg.t0; t < sg.t1 && ok; ++t) {
                    const bool switch_first = have_prev && t == sg.t0;
                    if (switch_first) ok = put_v(prev_row0, prev_t);
                    if (ok) ok = put_k(rb.kv_row0, t);
                    if (ok && have_prev && !switch_first) ok = put_v(prev_row0, prev_t);
                    have_prev = true;
                    prev_row0 = rb.kv_row0;
                    prev_t = t;
                }
            }
            if (ok && have_prev) ok = put_v(prev_row0, prev_t);
            for (int i = 0; i < C::NSLOT; ++i) drain_bar(bar(C::B_RFULL + i), issued[i], p.timeout_cycles);
        }
        // ------------------------------------------------------------ Q producer
        else if (warp == 1 && lane == 0) {
            const uint64_t pol_q = ptx::policy_evict_last();
            SegWalker wk;
            wk.init(p, misc->span, cta);
            Seg sg;
            int seg_i = 0;
            uint32_t q_issued = 0;
            while (wk.next(p, sg)) {
                if (sg.t1 <= sg.t0) continue;
                const RB rb = rb_of(p, sg.w);
                if (!wait_bar(bar(C::B_QEMPTY), (seg_i & 1) ^ 1, wmisc, p)) break;
                ptx::mbar_arrive_expect_tx(bar(C::B_QFULL), C::NBOX * p.q_box_rows * 128);
                ++q_issued;
                for (int bx = 0; bx < C::NBOX; ++bx)
                    ptx::tma_load_2d(sbase + C::OFF_Q + bx * C::Q_BOX, &tm_q, bx * 64, static_cast<int>(rb.q_row0),
                                     bar(C::B_QFULL), pol_q);
                ++seg_i;
            }
            drain_bar(bar(C::B_QFULL), q_issued, p.timeout_cycles);
        }
        // ------------------------------------------------------------ MMA issuer
        else if (warp == 2 && lane == 0) {
            SegWalker wk;
            wk.init(p, misc->span, cta);
            Seg sg;
            int seg_i = 0;
            uint32_t g = 0, seq = 0;
            bool ok = true;
            const uint32_t tm_o = tmem + C::TM_O;
            // next ring chunk, waited for
            auto take = [&](int& s) -> bool {
                s = static_cast<int>(seq % C::NSLOT);
                if (!wait_bar(bar(C::B_RFULL + s), (seq / C::NSLOT) & 1, wmisc, p)) return false;
                ptx::tc_fence_after();
                return true;
            };
            auto issue_s = [&](uint32_t gg, uint32_t qbase, bool last_of_seg) -> bool {
                const uint32_t d = tmem + C::TM_S + 128u * (gg & 1u);
                for (int c = 0; c < C::NBOX; ++c) {
                    int s;
                    if (!take(s)) return false;
                    const uint32_t kb = sbase + C::OFF_RING + s * C::CHUNK;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = ptx::umma_desc_sw128(qbase + c * C::Q_BOX + kk * 32, 16, 1024);
                        const uint64_t bd = ptx::umma_desc_sw128(kb + kk * 32, 16, 1024);
                        ptx::umma_bf16_ss(d, ad, bd, C::IDESC_S, (c > 0 || kk > 0) ? 1u : 0u);
                    }
                    ptx::umma_commit(bar(C::B_REMPTY + s));
                    ++seq;
                }
                ptx::umma_commit(bar(C::B_SFULL + (gg & 1u)));
                if (last_of_seg) ptx::umma_commit(bar(C::B_QEMPTY));
                return true;
            };
            // O[:, 64v .. 64v+63] (+)= P(gg) V_v(gg) for this CTA's V chunks v
            auto issue_pv = [&](uint32_t gg, bool first, int seg) -> bool {
                if (!wait_bar(bar(C::B_PFULL + (gg & 1u)), (gg >> 1) & 1u, wmisc, p)) return false;
                if (first && seg > 0 && !wait_bar(bar(C::B_OFREE), (seg - 1) & 1, wmisc, p)) return false;
                ptx::tc_fence_after();
                const uint32_t a = tmem + C::TM_S + 128u * (gg & 1u) + 64u;
                for (int v = 0; v < C::VCH; ++v) {
                    int s;
                    if (!take(s)) return false;
                    const uint32_t vb = sbase + C::OFF_RING + s * C::CHUNK;
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk) {
                        const uint64_t bd = ptx::umma_desc_sw128(vb + kk * 2048, C::CHUNK, 1024);
                        ptx::umma_bf16_ts(tm_o + v * 64, a + kk * 8, bd, C::IDESC_PV, (kk > 0 || !first) ? 1u : 0u);
                    }
                    ptx::umma_commit(bar(C::B_REMPTY + s));
                    ++seq;
                }
                ptx::umma_commit(bar(C::B_ODONE + (gg & 1u)));
                return true;
            };
            bool have_prev = false, prev_first = false;
            uint32_t prev_g = 0;
            int prev_seg = 0;
            while (ok && wk.next(p, sg)) {
                if (sg.t1 <= sg.t0) continue;
                // the previous segment's last PV goes out before this segment's Q is awaited
                if (have_prev) {
                    ok = issue_pv(prev_g, prev_first, prev_seg);
                    if (!ok) break;
                    have_prev = false;
                }
                ok = wait_bar(bar(C::B_QFULL), seg_i & 1, wmisc, p);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t qbase = sbase + C::OFF_Q;
                for (int t = sg.t0; t < sg.t1 && ok; ++t, ++g) {
                    ok = issue_s(g, qbase, t == sg.t1 - 1);
                    if (!ok) break;
                    if (have_prev) {
                        ok = issue_pv(prev_g, prev_first, prev_seg);
                        if (!ok) break;
                    }
                    have_prev = true;
                    prev_g = g;
                    prev_first = (t == sg.t0);
                    prev_seg = seg_i;
                }
                ++seg_i;
            }
            if (ok && have_prev) ok = issue_pv(prev_g, prev_first, prev_seg);
            // every MMA must retire before TMEM is released
            ptx::umma_commit(bar(C::B_FINAL));
            drain_bar(bar(C::B_FINAL), 1, p.timeout_cycles);
        }
        // ------------------------------------------------------------ publisher
        // For each split segment: once the softmax warps have written its partial
        // rows, make them visible GPU-wide and count this CTA's piece.
        else if (warp == 3 && lane == 0 && p.mode == 0) {
            SegWalker wk;
            wk.init(p, misc->span, cta);
            Seg sg;
            int j = 0;
            while (j < 2 && wk.next(p, sg)) {
                if (sg.kind != 1) continue;
                if (!wait_bar(bar(C::B_MJOB + j), 0, wmisc, p)) break;
                __threadfence();
                atomicAdd(wide_counters(p, sg.w, ho, C::DSPLIT), 1);
                ++j;
            }
        }
    }
    // ---------------------------------------------------------------- softmax / epilogue / merge
    else {
        const int quad = warp & 3;
        const int lrow = quad * 32 + lane;  // TMEM lane = row of the tile
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const int stid = threadIdx.x - 128;
        uint32_t xph = 0;
        auto xsync = [&]() -> bool {  // the four softmax warps, bounded
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
        bool ok = true;
        int njob = 0;
        constexpr int HD = C::DO;  // O columns of this CTA

        while (ok && wk.next(p, sg)) {
            const RB rb = rb_of(p, sg.w);
            const bool valid = lrow < rb.rows_valid;
            const int rp = rb.qt * BM + lrow;  // packed row inside the unit
            const int hl = valid ? rp / p.Tq : 0;
            const int i = valid ? rp % p.Tq : 0;
            int limit = p.causal ? (sg.n - p.Tq + i) : (sg.n - 1);
            if (limit > sg.n - 1) limit = sg.n - 1;
            if (!valid) limit = -1;
            const int h = rb.g * p.G + hl;
            const bool active = quad * 32 < rb.rows_valid;
            const bool nonempty = sg.t1 > sg.t0;

            float m_ref = -INFINITY;  // log2-domain reference max of the P values
            float l_sum = 0.f;

            for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                ok = wait_bar(bar(C::B_SFULL + (g & 1u)), (g >> 1) & 1u, wmisc, p);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ptx::tc_fence_after();
                const bool first = (t == sg.t0);
                float alpha = 1.f;
                const uint32_t ts = tmem + lane_off + C::TM_S + 128u * (g & 1u);
                if (active) {
                    float s[C::BN];
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
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < C::BN; c += 4) {
                        m4[0] = fmaxf(m4[0], s[c]);
                        m4[1] = fmaxf(m4[1], s[c + 1]);
                        m4[2] = fmaxf(m4[2], s[c + 2]);
                        m4[3] = fmaxf(m4[3], s[c + 3]);
                    }
                    const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * p.scale_log2;
                    if (first) {
                        m_ref = mt;
                    } else if (mt > m_ref + RESCALE_THRESHOLD) {
                        alpha = ptx::ex2(m_ref - mt);
                        m_ref = mt;
                    }
                    // P = 2^(s*scale*log2e - m) as bf16 over S's upper 64 columns
                    const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
                    float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int c = 0; c < C::BN / 32; ++c) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float a = ptx::ex2(fmaf(s[c * 32 + 2 * j], p.scale_log2, neg_m));
                            const float b = ptx::ex2(fmaf(s[c * 32 + 2 * j + 1], p.scale_log2, neg_m));
                            rs4[(2 * j) & 3] += a;
                            rs4[(2 * j + 1) & 3] += b;
                            pk[j] = pack_bf16x2(a, b);
                        }
                        ptx::tmem_st16(ts + 64 + c * 16, pk);
                    }
                    l_sum = l_sum * alpha + ((rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
                }
                // lazy rescale of O: only when some row's max grew by more than 2^8
                if (!first && __any_sync(0xffffffffu, alpha != 1.f)) {
                    bool okw = wait_bar(bar(C::B_ODONE + ((g - 1) & 1u)), ((g - 1) >> 1) & 1u, wmisc, p);
                    okw = __all_sync(0xffffffffu, okw);
                    if (!okw) {
                        ok = false;
                    } else {
                        ptx::tc_fence_after();
                        const uint32_t to = tmem + lane_off + C::TM_O;
#pragma unroll 1
                        for (int c = 0; c < HD / 32; ++c) {
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
                // padded key rows of V reach the MMA as zeros (0 * NaN = NaN); the tile
                // holding them is the last of its segment, so its V chunks sit at a
                // known place in the ring
                if ((t + 1) * C::BN > sg.n) {
                    const uint32_t vs = C::v_seq_last_of_segment(g);
                    int z0 = sg.n - t * C::BN;
                    z0 = z0 < 0 ? 0 : z0;
                    for (int v = 0; v < C::VCH && ok; ++v) {
                        const uint32_t sq = vs + v;
                        const int s = static_cast<int>(sq % C::NSLOT);
                        // the slot's previous chunk may still be in flight: wait for its
                        // release first, so that the fill wait below is for this chunk's
                        // phase and not one two phases back (same parity)
                        bool okv = wait_bar(bar(C::B_REMPTY + s), ((sq / C::NSLOT) & 1) ^ 1, wmisc, p);
                        okv = okv && wait_bar(bar(C::B_RFULL + s), (sq / C::NSLOT) & 1, wmisc, p);
                        okv = __all_sync(0xffffffffu, okv);
                        if (!okv) { ok = false; break; }
                        uint8_t* vt = smem + C::OFF_RING + s * C::CHUNK;
                        for (int q = stid; q < (C::BN - z0) * 8; q += NSOFT_W)
                            *reinterpret_cast<uint4*>(vt + (z0 + (q >> 3)) * 128 + (q & 7) * 16) = make_uint4(0, 0, 0, 0);
                    }
                    if (!ok) break;
                    ptx::fence_proxy_async_smem();
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::B_PFULL + (g & 1u)));
            }
            if (!ok) break;

            // ------------------------------------------------ segment epilogue
            if (nonempty) {
                ok = wait_bar(bar(C::B_ODONE + ((g - 1) & 1u)), ((g - 1) >> 1) & 1u, wmisc, p);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ptx::tc_fence_after();
            }
            float o_scale = 0.f, lse_v = -INFINITY;
            if (nonempty) {
                if (sg.kind == 0) {
                    const float sk = (p.sink != nullptr && valid) ? __ldg(p.sink + h) * LOG2E : -INFINITY;
                    const float M = fmax_nan(m_ref, sk);
                    if (M != -INFINITY) {
                        const float a = pos_or_nan(l_sum) ? ptx::ex2(m_ref - M) : 0.f;
                        const float lt = l_sum * a + ((sk != -INFINITY) ? ptx::ex2(sk - M) : 0.f);
                        if (pos_or_nan(lt)) {
                            o_scale = a / lt;
                            lse_v = (M + __log2f(lt)) * LN2;
                        }
                    }
                } else if (pos_or_nan(l_sum)) {
                    o_scale = 1.f / l_sum;
                    lse_v = (m_ref + __log2f(l_sum)) * LN2;
                }
            }
            const long long fr = rb.q_row0 + lrow;  // flat row (b*Hq + h)*Tq + i when valid
            const uint32_t to = tmem + lane_off + C::TM_O;
            if (sg.kind == 0) {
                __nv_bfloat16* dst = p.out + fr * C::D + ho * C::DO;
                if (active) {
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t r[32];
                        ptx::tmem_ld32(to + c * 32, r);
                        ptx::tmem_wait_ld();
                        if (valid) {
                            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                d4[j] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * j]) * o_scale, __uint_as_float(r[8 * j + 1]) * o_scale),
                                                   pack_bf16x2(__uint_as_float(r[8 * j + 2]) * o_scale, __uint_as_float(r[8 * j + 3]) * o_scale),
                                                   pack_bf16x2(__uint_as_float(r[8 * j + 4]) * o_scale, __uint_as_float(r[8 * j + 5]) * o_scale),
                                                   pack_bf16x2(__uint_as_float(r[8 * j + 6]) * o_scale, __uint_as_float(r[8 * j + 7]) * o_scale));
                        }
                    }
                }
                if (valid && ho == 0 && p.lse != nullptr) p.lse[fr] = lse_v;
            } else {
                // kind 1: this CTA's stream-K slot, float4 column groups of BM rows each;
                // kind 2: the public [B,Hq,Tq,S,d] layout
                float4* d4;
                long long jstride;  // float4s between consecutive column groups
                float* dl;
                if (sg.kind == 1) {
                    const long long slot = static_cast<long long>(sg.slot) * C::DSPLIT + ho;
                    d4 = reinterpret_cast<float4*>(p.part_o) + slot * C::GJ * BM + lrow;
                    jstride = BM;
                    dl = p.part_lse + slot * BM + lrow;
                } else {
                    d4 = reinterpret_cast<float4*>(p.part_o + (fr * p.num_splits + sg.slot) * C::D + ho * C::DO);
                    jstride = 1;
                    dl = p.part_lse + fr * p.num_splits + sg.slot;
                }
                if (active) {
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t r[32];
                        if (nonempty) {
                            ptx::tmem_ld32(to + c * 32, r);
                            ptx::tmem_wait_ld();
                        }
                        if (valid) {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                                if (nonempty)
                                    v4 = make_float4(__uint_as_float(r[4 * j]) * o_scale, __uint_as_float(r[4 * j + 1]) * o_scale,
                                                     __uint_as_float(r[4 * j + 2]) * o_scale, __uint_as_float(r[4 * j + 3]) * o_scale);
                                __stcg(d4 + (c * 8 + j) * jstride, v4);
                            }
                        }
                    }
                }
                if (valid && (sg.kind == 1 || ho == 0)) __stcg(dl, lse_v);
            }
            // O is read: the next segment's first PV may overwrite it
            if (nonempty) {
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::B_OFREE));
            }
            if (sg.kind == 1 && njob < 2) {
                // every softmax thread's partial rows are written: hand the piece to the publisher
                if (!xsync()) { ok = false; break; }
                if (stid == 0) {
                    misc->jobs[njob] = sg;
                    ptx::mbar_arrive(bar(C::B_MJOB + njob));
                }
                ++njob;
            }
        }

        // ------------------------------------------------ merges
        // Each split row-block this CTA holds a piece of is merged by all of its
        // pieces' CTAs together: each takes a range of O's column groups for every
        // row, stages every piece's block of those columns (and the pieces' lse)
        // in its now idle shared memory with one bulk copy per piece, and writes
        // the merged columns.
        uint32_t mph = 0;  // merge-barrier phases used
        for (int j = 0; ok && j < njob; ++j) {
            const Seg sm = misc->jobs[j];
            const RB rb = rb_of(p, sm.w);
            const long long tot = misc->span.tot;
            const int c_first = cta_of(sm.pw, tot, NC);
            const int c_last = cta_of(sm.pw + sm.ntiles - 1, tot, NC);
            const bool c0_first = span_begin(c_first, tot, NC) == sm.pw;
            int nc = 0, kme = 0;
            for (int cc = c_first; cc <= c_last; ++cc) {
                const bool has = span_begin(cc, tot, NC) < span_begin(cc + 1, tot, NC);
                if (has && cc < cta) ++kme;
                nc += has ? 1 : 0;
            }
            const int rows = rb.rows_valid;
            const int j0 = (kme * C::GJ) / nc, j1 = ((kme + 1) * C::GJ) / nc;  // this CTA's column groups
            int* ctr = wide_counters(p, sm.w, ho, C::DSPLIT);
            // wait until every piece is published
            if (stid == 0) {
                const long long t0 = clock64();
                while (ld_acquire(ctr) < nc) {
                    if (misc->abort) break;
                    if (clock64() - t0 > p.timeout_cycles) {
                        atomicCAS(p.err, 0, DEV_ERR_TIMEOUT);
                        misc->abort = 1;
                        break;
                    }
                }
                __threadfence();
            }
            // the slots of the pieces, in piece order
            if (warp == 4) {
                int n = 0;
                for (int base = c_first; base <= c_last; base += 32) {
                    const int cc = base + lane;
                    const bool has = cc <= c_last && span_begin(cc, tot, NC) < span_begin(cc + 1, tot, NC);
                    const unsigned m = __ballot_sync(0xffffffffu, has);
                    const int k = n + __popc(m & ((1u << lane) - 1u));
                    if (has && k < kWideSlotCap)
                        misc->mslot[k] = static_cast<int>(merge_slot(cc, c_first, c0_first) * C::DSPLIT + ho);
                    n += __popc(m);
                }
            }
            if (!xsync()) { ok = false; break; }
            if (misc->abort) { ok = false; break; }
            const float4* part4 = reinterpret_cast<const float4*>(p.part_o);
            const int r = stid;  // every thread owns one row of the tile
            const int hr = rb.g * p.G + (rb.qt * BM + (r < rows ? r : 0)) / p.Tq;
            const float sk = (p.sink != nullptr) ? __ldg(p.sink + hr) : -INFINITY;
            if (nc <= kWideStageMax) {
                // column groups per staging round: every piece's block of them fits
                const int fit = (C::STAGE_END - C::STAGE_O) / (nc * BM * 16);
                float* lse_st = reinterpret_cast<float*>(smem + C::STAGE_LSE);
                const float4* o_st = reinterpret_cast<const float4*>(smem + C::STAGE_O);
                bool first_round = true;
                for (int a = j0; ok && (a < j1 || first_round); a += fit) {
                    const int b = (a + fit < j1) ? a + fit : j1;
                    const int ncg = b - a;  // may be 0: the round still stages the lse
                    if (stid == 0) {
                        const uint32_t bytes = nc * ncg * BM * 16 + (first_round ? nc * BM * 4 : 0);
                        ptx::mbar_arrive_expect_tx(bar(C::B_MERGE), bytes);
                        for (int k = 0; k < nc; ++k) {
                            const long long sl = misc->mslot[k];
                            if (first_round)
                                ptx::bulk_load(sbase + C::STAGE_LSE + k * BM * 4, p.part_lse + sl * BM, BM * 4, bar(C::B_MERGE));
                            if (ncg > 0)
                                ptx::bulk_load(sbase + C::STAGE_O + k * ncg * BM * 16, part4 + (sl * C::GJ + a) * BM,
                                               ncg * BM * 16, bar(C::B_MERGE));
                        }
                    }
                    ok = wait_bar(bar(C::B_MERGE), mph & 1, wmisc, p);
                    ++mph;
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    if (first_round) {
                        // lse of this thread's row over the pieces (the sink enters once,
                        // here), then the pieces' weights in place of their lse
                        float mx = sk;
                        for (int k = 0; k < nc; ++k) mx = fmax_nan(mx, lse_st[k * BM + r]);
                        float z = 0.f;
                        if (mx != -INFINITY) {
                            for (int k = 0; k < nc; ++k) z += __expf(lse_st[k * BM + r] - mx);
                            if (sk != -INFINITY) z += __expf(sk - mx);
                        }
                        const float lt = (mx != -INFINITY && pos_or_nan(z)) ? mx + __logf(z) : -INFINITY;
                        for (int k = 0; k < nc; ++k)
                            lse_st[k * BM + r] = (lt != -INFINITY) ? __expf(lse_st[k * BM + r] - lt) : 0.f;
                        if (kme == 0 && ho == 0 && r < rows && p.lse != nullptr) p.lse[rb.q_row0 + r] = lt;
                        first_round = false;
                    }
                    // this thread's row, column groups a .. b
                    if (r < rows) {
                        __nv_bfloat16* orow = p.out + (rb.q_row0 + r) * C::D + ho * C::DO;
                        for (int jj = 0; jj < ncg; ++jj) {
                            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                            for (int k = 0; k < nc; ++k) {
                                const float w = lse_st[k * BM + r];
                                const float4 x = o_st[(k * ncg + jj) * BM + r];
                                acc.x += w * x.x;
                                acc.y += w * x.y;
                                acc.z += w * x.z;
                                acc.w += w * x.w;
                            }
                            *reinterpret_cast<uint2*>(orow + (a + jj) * 4) =
                                make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
                        }
                    }
                    // the staging area is rewritten by the next round
                    if (!xsync()) { ok = false; break; }
                    if (a >= j1) break;
                }
                if (!ok) break;
            } else {
                // many pieces: read them in place
                auto slot_of = [&](int k) -> long long {
                    if (nc <= kWideSlotCap) return misc->mslot[k];
                    int seen = 0;
                    for (int cc = c_first; cc <= c_last; ++cc) {
                        if (!(span_begin(cc, tot, NC) < span_begin(cc + 1, tot, NC))) continue;
                        if (seen++ == k) return merge_slot(cc, c_first, c0_first) * C::DSPLIT + ho;
                    }
                    return 0;
                };
                float mx = sk;
                for (int k = 0; k < nc; ++k) mx = fmax_nan(mx, __ldcg(p.part_lse + slot_of(k) * BM + r));
                float z = 0.f;
                if (mx != -INFINITY) {
                    for (int k = 0; k < nc; ++k) z += __expf(__ldcg(p.part_lse + slot_of(k) * BM + r) - mx);
                    if (sk != -INFINITY) z += __expf(sk - mx);
                }
                const float lt = (mx != -INFINITY && pos_or_nan(z)) ? mx + __logf(z) : -INFINITY;
                if (kme == 0 && ho == 0 && r < rows && p.lse != nullptr) p.lse[rb.q_row0 + r] = lt;
                if (r < rows) {
                    __nv_bfloat16* orow = p.out + (rb.q_row0 + r) * C::D + ho * C::DO;
                    for (int jj = j0; jj < j1; ++jj) {
                        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int k = 0; k < nc && lt != -INFINITY; ++k) {
                            const long long sl = slot_of(k);
                            const float w = __expf(__ldcg(p.part_lse + sl * BM + r) - lt);
                            const float4 x = __ldcg(part4 + (sl * C::GJ + jj) * BM + r);
                            acc.x += w * x.x;
                            acc.y += w * x.y;
                            acc.z += w * x.z;
                            acc.w += w * x.w;
                        }
                        *reinterpret_cast<uint2*>(orow + jj * 4) =
                            make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
                    }
                }
            }
            // this piece's merge is done; the last one leaves the counters at zero
            if (!xsync()) { ok = false; break; }
            if (stid == 0 && atomicAdd(ctr + 1, 1) == nc - 1) {
                ctr[0] = 0;
                ctr[1] = 0;
            }
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
