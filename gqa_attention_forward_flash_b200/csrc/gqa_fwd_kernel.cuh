// gqa_fwd_kernel.cuh -- sm_100a kernels of the GQA attention forward.
//
// One CTA (6 warps) streams the K/V tiles of one KV head once for a block of
// BM = 128 "packed" query rows: the G query heads that share the KV head times
// their Tq rows (AstrAI commit log, head-packing commit: K/V tiles stream once
// per block instead of once per q head).  Roles:
//   warp 0      TMA producer: Q tile per segment, ring of K and V tiles
//   warp 1      TMEM owner and single-thread tcgen05 MMA issuer:
//                 S = Q K^T into one of two TMEM S buffers,
//                 O += P V into the TMEM O accumulator
//   warps 2..5  softmax / correction / epilogue, one packed row per thread:
//                 logical-length + causal mask by selection, online (m, l)
//                 carry with lazy rescale of O, P -> bf16 into shared memory,
//                 final O / l (or a normalised partial + lse) to global memory
// (nvfp4-megamoe-kernel dsv4/kernels/attention commit log: multi-tile commit for
// the online softmax over KV tiles, prefill commits for the TMEM row/lane
// mapping, epilogue commits for TMEM -> registers -> global.)
//
// Work split.  Row-block w = (unit u = (b, kv head), q-tile qt) owns a key
// range of nkv(w) tiles of BN keys.  All tiles of all row-blocks are laid out
// in one flat order and cut into NC equal contiguous spans, one per CTA
// ("stream-K"): every CTA gets the same number of tiles whatever the lengths.
// A row-block finished inside one CTA is written straight to `out`; one cut by
// span boundaries leaves normalised fp32 partials in per-CTA slots, merged by
// the LSE combine kernel (AstrAI commit log: split-KV scratch commit;
// kernbench2 benches commit log: associative (m, l, O) merge).
#pragma once
#include <cuda_bf16.h>
#include <cuda.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace gqa {

constexpr int BM = 128;          // packed query rows per tile = TMEM lanes
constexpr int NUM_THREADS = 192; // 6 warps
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

// device error codes (same values as gqa_status)
constexpr int DEV_ERR_TIMEOUT = -6;
constexpr int DEV_ERR_KVLEN = -8;

struct Params {
    int B, Hq, Hkv, Tq, Tkv, d;
    int G, R, QT, U;      // R = G*Tq rows per unit, QT = ceil(R/BM) q-tiles, U = B*Hkv units
    long long W;          // row-blocks = U*QT
    int causal;
    int BN;               // keys per tile (set by the launcher to the kernel's BN)
    float scale_log2;     // scale * log2(e)
    const int* kv_lens;   // [B] or null
    const float* sink;    // [Hq] or null
    __nv_bfloat16* out;   // [B,Hq,Tq,d]
    float* lse;           // [B,Hq,Tq] or null
    int mode;             // 0: stream-K (direct + slots); 1: uniform splits (partials only)
    int num_splits;       // mode 1
    float* part_o;        // mode 0: [2*NC][BM][d] slots; mode 1: [B,Hq,Tq,S,d]
    float* part_lse;      // mode 0: [2*NC][BM];      mode 1: [B,Hq,Tq,S]
    long long* meta;      // mode 0: [NC][4] per-CTA combine record
    int* err;             // device error word
    long long timeout_cycles;
    int q_box_rows;       // rows of one Q TMA box: min(BM, B*Hq*Tq)
    int kv_box_rows;      // rows of one K/V TMA box: min(BN, B*Hkv*Tkv)
};

// ------------------------------------------------------------------ schedule
// These run on host (tests, planning) and device alike.

__host__ __device__ inline int clamp_len(int n, int Tkv, bool* bad) {
    if (n < 0) { if (bad) *bad = true; return 0; }
    if (n > Tkv) { if (bad) *bad = true; return Tkv; }
    return n;
}

// Leading key positions any row of q-tile qt may see (bottom-right causal).
__host__ __device__ inline int qtile_extent(const Params& p, int qt, int n) {
    if (!p.causal) return n;
    const int a = qt * BM;
    const int e = (p.R < a + BM ? p.R : a + BM) - 1;
    const int imax = (a / p.Tq != e / p.Tq) ? p.Tq - 1 : e % p.Tq;
    const int ext = n - p.Tq + imax + 1;
    return ext < 0 ? 0 : ext;
}

// Tiles of a row-block; at least one, so that a row-block with no visible key
// is still visited (its one tile is fully masked and it writes O = 0).
__host__ __device__ inline int qtile_ntiles(const Params& p, int qt, int n) {
    const int ext = qtile_extent(p, qt, n);
    const int t = (ext + p.BN - 1) / p.BN;
    return t < 1 ? 1 : t;
}

// Flat index -> owning CTA (spans are [floor(c*tot/NC), floor((c+1)*tot/NC))).
__host__ __device__ inline int cta_of(long long x, long long tot, int NC) {
    return static_cast<int>(((x + 1) * NC - 1) / tot);
}
__host__ __device__ inline long long span_begin(int c, long long tot, int NC) {
    return (static_cast<long long>(c) * tot) / NC;
}

struct Seg {
    int w;        // row-block (< 2^31 is checked on the host)
    int t0, t1;   // tile range inside the row-block
    int ntiles;   // nkv(w)
    int n;        // logical length of the row-block's batch
    int kind;     // 0: direct, 1: stream-K slot, 2: uniform split
    int slot;     // slot (kind 1) or split index (kind 2)
};

__device__ __forceinline__ int load_len(const Params& p, int b) {
    if (p.kv_lens == nullptr) return p.Tkv;
    bool bad = false;
    int n = clamp_len(__ldg(p.kv_lens + b), p.Tkv, &bad);
    if (bad) atomicCAS(p.err, 0, DEV_ERR_KVLEN);
    return n;
}

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Tiles in one unit of a batch with logical length n (all lanes of a warp call).
__device__ long long unit_tiles_warp(const Params& p, int n) {
    if (!p.causal) {
        int t = (n + p.BN - 1) / p.BN;
        return static_cast<long long>(p.QT) * (t < 1 ? 1 : t);
    }
    const int lane = threadIdx.x & 31;
    long long acc = 0;
    for (int qt = lane; qt < p.QT; qt += 32) acc += qtile_ntiles(p, qt, n);
    return warp_sum_ll(acc);
}

struct SpanStart {
    long long tot, p0, p1;
    int w, t;
};

// One full warp: total tiles, this CTA's span and the (row-block, tile) where it starts.
__device__ void plan_span(const Params& p, int c, int NC, SpanStart* out) {
    const int lane = threadIdx.x & 31;
    long long tot = 0;
    if (p.kv_lens == nullptr) {
        tot = static_cast<long long>(p.U) * unit_tiles_warp(p, p.Tkv);
    } else {
        for (int b = 0; b < p.B; ++b) tot += p.Hkv * unit_tiles_warp(p, load_len(p, b));
    }
    const long long p0 = span_begin(c, tot, NC), p1 = span_begin(c + 1, tot, NC);
    int w = 0, t = 0;
    if (p0 < p1) {
        // batch, then unit, then q-tile containing flat index p0
        long long acc = 0;
        int b = 0, n = p.Tkv;
        long long per_unit = 0;
        if (p.kv_lens == nullptr) {
            per_unit = unit_tiles_warp(p, n);
            b = static_cast<int>(p0 / (per_unit * p.Hkv));
            acc = static_cast<long long>(b) * per_unit * p.Hkv;
        } else {
            for (b = 0; b < p.B; ++b) {
                n = load_len(p, b);
                per_unit = unit_tiles_warp(p, n);
                if (p0 < acc + per_unit * p.Hkv) break;
                acc += per_unit * p.Hkv;
            }
        }
        const long long in_b = p0 - acc;
        const int ul = static_cast<int>(in_b / per_unit);
        long long rem = in_b - static_cast<long long>(ul) * per_unit;
        const int u = b * p.Hkv + ul;
        int qt = 0;
        if (!p.causal) {
            int nt = (n + p.BN - 1) / p.BN;
            nt = nt < 1 ? 1 : nt;
            qt = static_cast<int>(rem / nt);
            rem -= static_cast<long long>(qt) * nt;
        } else {
            // warp scan over q-tiles, 32 at a time
            for (int base = 0; base < p.QT; base += 32) {
                const int q = base + lane;
                long long cnt = q < p.QT ? qtile_ntiles(p, q, n) : 0;
                long long inc = cnt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    long long y = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += y;
                }
                const long long chunk_total = __shfl_sync(0xffffffffu, inc, 31);
                if (rem < chunk_total) {
                    const unsigned hit = __ballot_sync(0xffffffffu, rem < inc);
                    const int L = __ffs(hit) - 1;
                    const long long before = __shfl_sync(0xffffffffu, inc - cnt, L);
                    qt = base + L;
                    rem -= before;
                    break;
                }
                rem -= chunk_total;
            }
        }
        w = u * p.QT + qt;
        t = static_cast<int>(rem);
    }
    if (lane == 0) {
        out->tot = tot;
        out->p0 = p0;
        out->p1 = p1;
        out->w = w;
        out->t = t;
    }
}

// Walks this CTA's segments (every role keeps its own copy; all see the same sequence).
struct SegWalker {
    int w, t;
    long long remaining;
    bool first;
    int c;

    __device__ void init_streamk(const SpanStart& s, int cta) {
        w = s.w;
        t = s.t;
        remaining = s.p1 - s.p0;
        first = true;
        c = cta;
    }
    // mode 0
    __device__ bool next(const Params& p, Seg& sg) {
        if (remaining <= 0) return false;
        const int u = w / p.QT, qt = w % p.QT;
        const int n = load_len(p, u / p.Hkv);
        const int nt = qtile_ntiles(p, qt, n);
        long long take = nt - t;
        if (take > remaining) take = remaining;
        sg.w = w;
        sg.t0 = t;
        sg.t1 = t + static_cast<int>(take);
        sg.ntiles = nt;
        sg.n = n;
        const bool full = (t == 0 && sg.t1 == nt);
        sg.kind = full ? 0 : 1;
        sg.slot = first ? 2 * c : 2 * c + 1;
        remaining -= take;
        first = false;
        ++w;
        t = 0;
        return true;
    }
};

// mode 1: CTA = (row-block, split); the single segment may be empty (t0 == t1).
__device__ inline void uniform_segment(const Params& p, int cta, Seg& sg) {
    const int S = p.num_splits;
    sg.w = cta / S;
    const int s = cta % S;
    const int u = sg.w / p.QT, qt = sg.w % p.QT;
    sg.n = load_len(p, u / p.Hkv);
    sg.ntiles = qtile_ntiles(p, qt, sg.n);
    sg.t0 = static_cast<int>((static_cast<long long>(s) * sg.ntiles) / S);
    sg.t1 = static_cast<int>((static_cast<long long>(s + 1) * sg.ntiles) / S);
    sg.kind = 2;
    sg.slot = s;
}

// ------------------------------------------------------------------ kernel config

template <int D_, int BN_, int ST_, int QBUF_>
struct FwdCfg {
    static constexpr int D = D_, BN = BN_, ST = ST_, QBUF = QBUF_;
    static_assert(D % 64 == 0 && D <= 256, "head dim");
    static_assert(BN == 64 || BN == 128, "key tile");
    static constexpr int NBOX = D / 64;                 // 64-column swizzle boxes per row
    static constexpr int Q_BOX = BM * 128;              // bytes of one Q box
    static constexpr int Q_BYTES = NBOX * Q_BOX;
    static constexpr int KV_BOX = BN * 128;
    static constexpr int KV_BYTES = NBOX * KV_BOX;      // one K (or V) tile
    static constexpr int P_BOX = BM * 128;
    static constexpr int P_BYTES = (BN / 64) * P_BOX;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QBUF * Q_BYTES;
    static constexpr int OFF_V = OFF_K + ST * KV_BYTES;
    static constexpr int OFF_P = OFF_V + ST * KV_BYTES;
    static constexpr int OFF_BAR = OFF_P + P_BYTES;
    // barrier indices
    static constexpr int B_QFULL = 0;
    static constexpr int B_QEMPTY = B_QFULL + QBUF;
    static constexpr int B_KFULL = B_QEMPTY + QBUF;
    static constexpr int B_KEMPTY = B_KFULL + ST;
    static constexpr int B_VFULL = B_KEMPTY + ST;
    static constexpr int B_VEMPTY = B_VFULL + ST;
    static constexpr int B_SFULL = B_VEMPTY + ST;   // 2
    static constexpr int B_SFREE = B_SFULL + 2;     // 2
    static constexpr int B_PFULL = B_SFREE + 2;
    static constexpr int B_ODONE = B_PFULL + 1;
    static constexpr int B_FINAL = B_ODONE + 1;
    static constexpr int NBAR = B_FINAL + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int MISC_BYTES = 64;
    static constexpr int SMEM_USED = OFF_MISC + MISC_BYTES;
    static constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack to align the base to 1024
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    // TMEM columns
    static constexpr uint32_t TM_O = 0;
    static constexpr uint32_t TM_S0 = 256;
    static constexpr uint32_t TM_COLS = 512;
    static constexpr uint32_t IDESC_S = ptx::umma_idesc_bf16_f32(BM, BN, false, false);
    static constexpr uint32_t IDESC_PV = ptx::umma_idesc_bf16_f32(BM, D, false, true);
};

struct Misc {
    uint32_t tmem_base;
    volatile int abort;
    int pad0, pad1;
    SpanStart span;   // 40 bytes
};
static_assert(sizeof(Misc) <= 64, "misc block");

// Bounded wait; on expiry records GQA_ERR_TIMEOUT and raises the CTA abort flag.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, Misc* misc, const Params& p) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (misc->abort) return false;
        if (clock64() - t0 > p.timeout_cycles) {
            atomicCAS(p.err, 0, DEV_ERR_TIMEOUT);
            misc->abort = 1;
            return false;
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Row-block geometry shared by the roles.
struct RB {
    int b, g, qt;
    long long q_row0;   // first row in the 2-D [B*Hq*Tq, d] view of Q / out
    long long kv_row0;  // first row in the 2-D [B*Hkv*Tkv, d] view of K / V
    int rows_valid;     // packed rows of this q-tile that exist (<= BM)
};
__device__ __forceinline__ RB rb_of(const Params& p, int w) {
    RB r;
    const int u = w / p.QT;
    r.qt = w % p.QT;
    r.b = u / p.Hkv;
    r.g = u % p.Hkv;
    r.q_row0 = (static_cast<long long>(r.b) * p.Hq + static_cast<long long>(r.g) * p.G) * p.Tq +
               static_cast<long long>(r.qt) * BM;
    r.kv_row0 = static_cast<long long>(u) * p.Tkv;
    const int left = p.R - r.qt * BM;
    r.rows_valid = left < BM ? left : BM;
    return r;
}

template <class C>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gqa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
    Misc* misc = reinterpret_cast<Misc*>(smem + C::OFF_MISC);

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
        for (int i = 0; i < C::ST; ++i) {
            ptx::mbar_init(bar(C::B_KFULL + i), 1);
            ptx::mbar_init(bar(C::B_KEMPTY + i), 1);
            ptx::mbar_init(bar(C::B_VFULL + i), 1);
            ptx::mbar_init(bar(C::B_VEMPTY + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(C::B_SFULL + i), 1);
            ptx::mbar_init(bar(C::B_SFREE + i), 128);
        }
        ptx::mbar_init(bar(C::B_PFULL), 128);
        ptx::mbar_init(bar(C::B_ODONE), 1);
        ptx::mbar_init(bar(C::B_FINAL), 1);
        misc->abort = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tm_q);
        ptx::tma_prefetch_desc(&tm_k);
        ptx::tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr(&misc->tmem_base), C::TM_COLS);
        ptx::tmem_relinquish();
    }
    if (p.mode == 0 && warp == 0) plan_span(p, cta, NC, &misc->span);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    // ---------------------------------------------------------------- producer
    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_q = ptx::policy_evict_last();
            const uint64_t pol_kv = (p.QT == 1) ? ptx::policy_evict_first() : ptx::policy_evict_normal();
            SegWalker wk;
            Seg sg;
            bool more;
            if (p.mode == 0) wk.init_streamk(misc->span, cta);
            int seg_i = 0;
            uint32_t g = 0;
            bool ok = true;
            bool single_done = false;
            uint32_t k_issued[C::ST], v_issued[C::ST], q_issued[C::QBUF];
            for (int i = 0; i < C::ST; ++i) k_issued[i] = v_issued[i] = 0;
            for (int i = 0; i < C::QBUF; ++i) q_issued[i] = 0;
            while (ok) {
                if (p.mode == 0) {
                    more = wk.next(p, sg);
                } else {
                    more = !single_done;
                    single_done = true;
                    if (more) uniform_segment(p, cta, sg);
                }
                if (!more) break;
                if (sg.t1 <= sg.t0) continue;  // empty split: nothing to load
                const RB rb = rb_of(p, sg.w);
                const int qb = seg_i % C::QBUF;
                ok = wait_bar(bar(C::B_QEMPTY + qb), ((seg_i / C::QBUF) & 1) ^ 1, misc, p);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(bar(C::B_QFULL + qb), C::NBOX * p.q_box_rows * 128);
                ++q_issued[qb];
                for (int bx = 0; bx < C::NBOX; ++bx)
                    ptx::tma_load_2d(sbase + C::OFF_Q + qb * C::Q_BYTES + bx * C::Q_BOX, &tm_q, bx * 64,
                                     static_cast<int>(rb.q_row0), bar(C::B_QFULL + qb), pol_q);
                for (int t = sg.t0; t < sg.t1 && ok; ++t, ++g) {
                    const int st = g % C::ST;
                    const uint32_t ph = ((g / C::ST) & 1) ^ 1;
                    const int y = static_cast<int>(rb.kv_row0 + static_cast<long long>(t) * C::BN);
                    ok = wait_bar(bar(C::B_KEMPTY + st), ph, misc, p);
                    if (!ok) break;
                    ptx::mbar_arrive_expect_tx(bar(C::B_KFULL + st), C::NBOX * p.kv_box_rows * 128);
                    ++k_issued[st];
                    for (int bx = 0; bx < C::NBOX; ++bx)
                        ptx::tma_load_2d(sbase + C::OFF_K + st * C::KV_BYTES + bx * C::KV_BOX, &tm_k,
                                         bx * 64, y, bar(C::B_KFULL + st), pol_kv);
                    ok = wait_bar(bar(C::B_VEMPTY + st), ph, misc, p);
                    if (!ok) break;
                    ptx::mbar_arrive_expect_tx(bar(C::B_VFULL + st), C::NBOX * p.kv_box_rows * 128);
                    ++v_issued[st];
                    for (int bx = 0; bx < C::NBOX; ++bx)
                        ptx::tma_load_2d(sbase + C::OFF_V + st * C::KV_BYTES + bx * C::KV_BOX, &tm_v,
                                         bx * 64, y, bar(C::B_VFULL + st), pol_kv);
                }
                ++seg_i;
            }
            // Never leave the CTA with copies in flight: wait (bounded) for the last
            // load issued into every stage and Q buffer, also after an abort.
            auto drain = [&](uint32_t b, uint32_t issued) {
                if (issued == 0) return;
                const uint32_t par = (issued - 1) & 1;
                const long long t0 = clock64();
                while (!ptx::mbar_try_wait(b, par) && clock64() - t0 < p.timeout_cycles) {}
            };
            for (int i = 0; i < C::ST; ++i) {
                drain(bar(C::B_KFULL + i), k_issued[i]);
                drain(bar(C::B_VFULL + i), v_issued[i]);
            }
            for (int i = 0; i < C::QBUF; ++i) drain(bar(C::B_QFULL + i), q_issued[i]);
        } else if (lane == 1 && p.mode == 0) {
            // Per-CTA combine record: this CTA starts a row-block it does not finish.
            const SpanStart s = misc->span;
            long long rec[4] = {-1, 0, 0, s.tot};
            if (s.p1 > s.p0) {
                SegWalker wk;
                wk.init_streamk(s, cta);
                Seg sg, last;
                int count = 0;
                while (wk.next(p, sg)) { last = sg; ++count; }
                if (count > 0 && last.t0 == 0 && last.t1 < last.ntiles) {
                    const long long pw = s.p1 - (last.t1 - last.t0);
                    rec[0] = last.w;
                    rec[1] = cta_of(pw + last.ntiles - 1, s.tot, NC);
                    rec[2] = last.slot;
                }
            }
            long long* m = p.meta + 4ll * cta;
            m[0] = rec[0];
            m[1] = rec[1];
            m[2] = rec[2];
            m[3] = rec[3];
        }
    }
    // ---------------------------------------------------------------- MMA issuer
    else if (warp == 1) {
        if (lane == 0) {
            SegWalker wk;
            Seg sg;
            bool more;
            if (p.mode == 0) wk.init_streamk(misc->span, cta);
            int seg_i = 0;
            uint32_t g = 0;
            bool ok = true;
            bool single_done = false;
            bool have_prev = false;     // a PV is pending for tile g-1
            bool prev_first = false;    // ... and it is the first tile of its segment
            const uint32_t tm_o = tmem + C::TM_O;

            auto issue_pv = [&](uint32_t gp, bool first_of_seg) -> bool {
                if (!wait_bar(bar(C::B_PFULL), gp & 1, misc, p)) return false;
                const int st = gp % C::ST;
                if (!wait_bar(bar(C::B_VFULL + st), (gp / C::ST) & 1, misc, p)) return false;
                ptx::tc_fence_after();
                const uint32_t pbase = sbase + C::OFF_P;
                const uint32_t vbase = sbase + C::OFF_V + st * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    const uint64_t ad = ptx::umma_desc_sw128(pbase + (kk >> 2) * C::P_BOX + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = ptx::umma_desc_sw128(vbase + kk * 2048, C::KV_BOX, 1024);
                    ptx::umma_bf16_ss(tm_o, ad, bd, C::IDESC_PV, (kk > 0 || !first_of_seg) ? 1u : 0u);
                }
                ptx::umma_commit(bar(C::B_ODONE));
                ptx::umma_commit(bar(C::B_VEMPTY + st));
                return true;
            };

            while (ok) {
                if (p.mode == 0) {
                    more = wk.next(p, sg);
                } else {
                    more = !single_done;
                    single_done = true;
                    if (more) uniform_segment(p, cta, sg);
                }
                if (!more) break;
                if (sg.t1 <= sg.t0) continue;
                const int qb = seg_i % C::QBUF;
                ok = wait_bar(bar(C::B_QFULL + qb), (seg_i / C::QBUF) & 1, misc, p);
                if (!ok) break;
                const uint32_t qbase = sbase + C::OFF_Q + qb * C::Q_BYTES;
                for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                    const int st = g % C::ST;
                    const int sb = g & 1;
                    ok = wait_bar(bar(C::B_KFULL + st), (g / C::ST) & 1, misc, p);
                    if (!ok) break;
                    if (g >= 2) {
                        ok = wait_bar(bar(C::B_SFREE + sb), ((g >> 1) - 1) & 1, misc, p);
                        if (!ok) break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t kbase = sbase + C::OFF_K + st * C::KV_BYTES;
                    const uint32_t tm_s = tmem + C::TM_S0 + sb * 128;
#pragma unroll
                    for (int kk = 0; kk < C::D / 16; ++kk) {
                        const uint32_t off = (kk & 3) * 32;
                        const uint64_t ad = ptx::umma_desc_sw128(qbase + (kk >> 2) * C::Q_BOX + off, 16, 1024);
                        const uint64_t bd = ptx::umma_desc_sw128(kbase + (kk >> 2) * C::KV_BOX + off, 16, 1024);
                        ptx::umma_bf16_ss(tm_s, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    ptx::umma_commit(bar(C::B_SFULL + sb));
                    ptx::umma_commit(bar(C::B_KEMPTY + st));
                    if (t == sg.t1 - 1) ptx::umma_commit(bar(C::B_QEMPTY + qb));
                    if (have_prev) {
                        ok = issue_pv(g - 1, prev_first);
                        if (!ok) break;
                    }
                    have_prev = true;
                    prev_first = (t == sg.t0);
                }
                ++seg_i;
            }
            if (ok && have_prev) ok = issue_pv(g - 1, prev_first);
            // make sure every MMA has retired before TMEM is released
            ptx::umma_commit(bar(C::B_FINAL));
            const long long t0 = clock64();
            while (!ptx::mbar_try_wait(bar(C::B_FINAL), 0) && clock64() - t0 < p.timeout_cycles) {}
        }
    }
    // ---------------------------------------------------------------- softmax / epilogue
    else {
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t tm_o = tmem + lane_off + C::TM_O;
        SegWalker wk;
        Seg sg;
        bool more;
        if (p.mode == 0) wk.init_streamk(misc->span, cta);
        uint32_t g = 0;
        bool ok = true;
        bool single_done = false;
        uint8_t* const p_smem = smem + C::OFF_P;

        while (ok) {
            if (p.mode == 0) {
                more = wk.next(p, sg);
            } else {
                more = !single_done;
                single_done = true;
                if (more) uniform_segment(p, cta, sg);
            }
            if (!more) break;
            const RB rb = rb_of(p, sg.w);
            const int rp = rb.qt * BM + row;           // packed row inside the unit
            const bool valid = row < rb.rows_valid;
            const int hl = valid ? rp / p.Tq : 0;      // head inside the group
            const int i = valid ? rp % p.Tq : 0;
            int limit = p.causal ? (sg.n - p.Tq + i) : (sg.n - 1);
            if (limit > sg.n - 1) limit = sg.n - 1;
            if (!valid) limit = -1;
            const int h = rb.g * p.G + hl;

            float m_ref = -INFINITY;  // log2-domain running max used for P
            float l_sum = 0.f;

            for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                const int sb = g & 1;
                ok = wait_bar(bar(C::B_SFULL + sb), (g >> 1) & 1, misc, p);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ptx::tc_fence_after();
                float s[C::BN];
                {
                    const uint32_t tm_s = tmem + lane_off + C::TM_S0 + sb * 128;
#pragma unroll
                    for (int c = 0; c < C::BN / 32; ++c) {
                        uint32_t r[32];
                        ptx::tmem_ld32(tm_s + c * 32, r);
#pragma unroll
                        for (int j = 0; j < 32; ++j) s[c * 32 + j] = __uint_as_float(r[j]);
                    }
                    ptx::tmem_wait_ld();
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(bar(C::B_SFREE + sb));

                // mask (select, never add: NaN + -inf would stay NaN) and row max
                const int lim = limit - t * C::BN;
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < C::BN; ++c) {
                    const float x = (c <= lim) ? s[c] * p.scale_log2 : -INFINITY;
                    s[c] = x;
                    mx = fmaxf(mx, x);
                }
                const bool first = (t == sg.t0);
                float alpha = 1.f;
                if (first) {
                    m_ref = mx;
                } else if (mx > m_ref + RESCALE_THRESHOLD) {
                    alpha = exp2f(m_ref - mx);
                    m_ref = mx;
                }
                const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;

                // the previous PV must be done: P buffer reuse and O rescale
                if (g >= 1) {
                    ok = wait_bar(bar(C::B_ODONE), (g - 1) & 1, misc, p);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    ptx::tc_fence_after();
                }
                if (!first && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                    for (int c = 0; c < C::D / 32; ++c) {
                        uint32_t r[32];
                        ptx::tmem_ld32(tm_o + c * 32, r);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
                        ptx::tmem_st32(tm_o + c * 32, r);
                    }
                    ptx::tmem_wait_st();
                }
                // padded key rows of the V tile must reach the MMA as zeros (0 * NaN = NaN)
                if ((t + 1) * C::BN > sg.n) {
                    const int st = g % C::ST;
                    ok = wait_bar(bar(C::B_VFULL + st), (g / C::ST) & 1, misc, p);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    int z0 = sg.n - t * C::BN;
                    z0 = z0 < 0 ? 0 : z0;
                    uint8_t* vt = smem + C::OFF_V + st * C::KV_BYTES;
                    const int chunks = (C::BN - z0) * C::NBOX * 8;  // 16-byte chunks
                    for (int q = threadIdx.x - 64; q < chunks; q += 128) {
                        const int r = z0 + q / (C::NBOX * 8);
                        const int rem = q % (C::NBOX * 8);
                        const int bx = rem / 8, ch = rem % 8;
                        *reinterpret_cast<uint4*>(vt + bx * C::KV_BOX + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
                    }
                }
                // P = exp2(x - m) -> bf16, written in the 128-byte-swizzled K-major image
                float rs = 0.f;
#pragma unroll
                for (int c8 = 0; c8 < C::BN / 8; ++c8) {
                    uint32_t pk[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float a = exp2f(s[c8 * 8 + 2 * j] - m_use);
                        const float b = exp2f(s[c8 * 8 + 2 * j + 1] - m_use);
                        pk[j] = pack_bf16x2(a, b);
                        rs += a + b;
                    }
                    const int bx = c8 >> 3;
                    const int ch = (c8 & 7) ^ (row & 7);
                    *reinterpret_cast<uint4*>(p_smem + bx * C::P_BOX + row * 128 + ch * 16) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
                l_sum = l_sum * alpha + rs;
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                ptx::mbar_arrive(bar(C::B_PFULL));
            }
            if (!ok) break;

            // ------------------------------------------------ segment epilogue
            float o_scale = 0.f, lse_v = -INFINITY;
            if (sg.t1 > sg.t0) {
                ok = wait_bar(bar(C::B_ODONE), (g - 1) & 1, misc, p);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ptx::tc_fence_after();
                if (sg.kind == 0) {
                    const float sk = (p.sink != nullptr && valid) ? __ldg(p.sink + h) * LOG2E : -INFINITY;
                    const float M = fmaxf(m_ref, sk);
                    if (M != -INFINITY) {
                        const float a = exp2f(m_ref - M);
                        const float lt = l_sum * a + exp2f(sk - M);
                        o_scale = a / lt;
                        lse_v = (M + log2f(lt)) * LN2;
                    }
                } else if (l_sum > 0.f) {
                    o_scale = 1.f / l_sum;
                    lse_v = (m_ref + log2f(l_sum)) * LN2;
                }
            }
            // destination of this row
            const long long fr = rb.q_row0 + row;  // flat row (b*Hq + h)*Tq + i when valid
            if (sg.kind == 0) {
                __nv_bfloat16* dst = p.out + fr * C::D;
#pragma unroll 1
                for (int c = 0; c < C::D / 32; ++c) {
                    uint32_t r[32];
                    if (sg.t1 > sg.t0) {
                        ptx::tmem_ld32(tm_o + c * 32, r);
                        ptx::tmem_wait_ld();
                    }
                    if (valid) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            pk[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * o_scale,
                                                __uint_as_float(r[2 * j + 1]) * o_scale);
                        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                        for (int j = 0; j < 4; ++j) d4[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                    }
                }
                if (valid && p.lse != nullptr) p.lse[fr] = lse_v;
            } else {
                float* dst;
                float* dl;
                if (sg.kind == 1) {
                    dst = p.part_o + (static_cast<long long>(sg.slot) * BM + row) * C::D;
                    dl = p.part_lse + static_cast<long long>(sg.slot) * BM + row;
                } else {
                    dst = p.part_o + (fr * p.num_splits + sg.slot) * C::D;
                    dl = p.part_lse + fr * p.num_splits + sg.slot;
                }
#pragma unroll 1
                for (int c = 0; c < C::D / 32; ++c) {
                    uint32_t r[32];
                    if (sg.t1 > sg.t0) {
                        ptx::tmem_ld32(tm_o + c * 32, r);
                        ptx::tmem_wait_ld();
                    }
                    if (valid) {
                        float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            float4 v4;
                            if (sg.t1 > sg.t0) {
                                v4 = make_float4(__uint_as_float(r[4 * j]) * o_scale, __uint_as_float(r[4 * j + 1]) * o_scale,
                                                 __uint_as_float(r[4 * j + 2]) * o_scale, __uint_as_float(r[4 * j + 3]) * o_scale);
                            } else {
                                v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                            }
                            d4[j] = v4;
                        }
                    }
                }
                if (valid) *dl = lse_v;
            }
            ptx::tc_fence_before();
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::TM_COLS);
    }
}

// ------------------------------------------------------------------ combine kernels

// Stream-K combine: block c merges the row-block that CTA c started but did not finish.
template <int D>
__global__ void __launch_bounds__(256)
gqa_combine_streamk_kernel(const Params p) {
    const int c = blockIdx.x;
    const int NC = gridDim.x;
    const long long* m = p.meta + 4ll * c;
    const long long w = m[0];
    if (w < 0) return;
    const int c_last = static_cast<int>(m[1]);
    const int slot0 = static_cast<int>(m[2]);
    const long long tot = m[3];
    if (w >= p.W || c_last < c || c_last >= NC || slot0 < 0 || slot0 >= 2 * NC || tot <= 0) {
        if (threadIdx.x == 0) atomicCAS(p.err, 0, DEV_ERR_TIMEOUT);
        return;
    }

    __shared__ int slots[512];
    __shared__ int nslots;
    __shared__ float row_lse[BM];
    if (threadIdx.x == 0) {
        int k = 0;
        slots[k++] = slot0;
        for (int cc = c + 1; cc <= c_last && k < 512; ++cc)
            if (span_begin(cc, tot, NC) < span_begin(cc + 1, tot, NC)) slots[k++] = 2 * cc;
        nslots = k;
    }
    __syncthreads();
    const int ns = nslots;
    const RB rb = rb_of(p, static_cast<int>(w));
    for (int r = threadIdx.x; r < rb.rows_valid; r += blockDim.x) {
        const int rp = rb.qt * BM + r;
        const int h = rb.g * p.G + rp / p.Tq;
        float L = (p.sink != nullptr) ? __ldg(p.sink + h) : -INFINITY;
        for (int k = 0; k < ns; ++k) L = fmaxf(L, p.part_lse[static_cast<long long>(slots[k]) * BM + r]);
        float lt = -INFINITY;
        if (L != -INFINITY) {
            float z = (p.sink != nullptr) ? __expf(__ldg(p.sink + h) - L) : 0.f;
            for (int k = 0; k < ns; ++k) z += __expf(p.part_lse[static_cast<long long>(slots[k]) * BM + r] - L);
            lt = L + __logf(z);
        }
        row_lse[r] = lt;
        if (p.lse != nullptr) p.lse[rb.q_row0 + r] = lt;
    }
    __syncthreads();
    constexpr int C4 = D / 4;
    for (int it = threadIdx.x; it < rb.rows_valid * C4; it += blockDim.x) {
        const int r = it / C4, c4 = it % C4;
        const float lt = row_lse[r];
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lt != -INFINITY) {
            for (int k = 0; k < ns; ++k) {
                const long long sl = slots[k];
                const float wgt = __expf(p.part_lse[sl * BM + r] - lt);
                if (wgt == 0.f) continue;
                const float4 o = *reinterpret_cast<const float4*>(p.part_o + (sl * BM + r) * D + 4 * c4);
                acc.x += wgt * o.x;
                acc.y += wgt * o.y;
                acc.z += wgt * o.z;
                acc.w += wgt * o.w;
            }
        }
        uint2 pk = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
        *reinterpret_cast<uint2*>(p.out + (rb.q_row0 + r) * D + 4 * c4) = pk;
    }
}

// Uniform combine (public entry): one warp per row, S partials laid out [rows, S, d].
__global__ void __launch_bounds__(256)
gqa_combine_uniform_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part, int S,
                           const float* __restrict__ sink, __nv_bfloat16* __restrict__ out,
                           float* __restrict__ lse, long long rows, int Hq, int Tq, int d) {
    extern __shared__ float wsm[];  // [8 warps][S]
    const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* wts = wsm + wib * S;
    const long long nwarps = static_cast<long long>(gridDim.x) * 8;
    for (long long row = static_cast<long long>(blockIdx.x) * 8 + wib; row < rows; row += nwarps) {
        const int h = static_cast<int>((row / Tq) % Hq);
        const float sk = (sink != nullptr) ? sink[h] : -INFINITY;
        float L = sk;
        for (int s = lane; s < S; s += 32) L = fmaxf(L, lse_part[row * S + s]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L = fmaxf(L, __shfl_xor_sync(0xffffffffu, L, o));
        float lt = -INFINITY;
        if (L != -INFINITY) {
            float z = 0.f;
            for (int s = lane; s < S; s += 32) z += __expf(lse_part[row * S + s] - L);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            if (sink != nullptr) z += __expf(sk - L);
            lt = L + __logf(z);
        }
        for (int s = lane; s < S; s += 32) wts[s] = (lt == -INFINITY) ? 0.f : __expf(lse_part[row * S + s] - lt);
        __syncwarp();
        for (int c4 = lane; c4 < d / 4; c4 += 32) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s = 0; s < S; ++s) {
                const float wgt = wts[s];
                if (wgt == 0.f) continue;
                const float4 o = *reinterpret_cast<const float4*>(o_part + (row * S + s) * d + 4 * c4);
                acc.x += wgt * o.x;
                acc.y += wgt * o.y;
                acc.z += wgt * o.z;
                acc.w += wgt * o.w;
            }
            uint2 pk = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
            *reinterpret_cast<uint2*>(out + row * d + 4 * c4) = pk;
        }
        if (lane == 0 && lse != nullptr) lse[row] = lt;
        __syncwarp();
    }
}

}  // namespace gqa
