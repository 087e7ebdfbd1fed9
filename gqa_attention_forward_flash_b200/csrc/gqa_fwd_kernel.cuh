// gqa_fwd_kernel.cuh -- sm_100a kernels of the GQA attention forward.
//
// One CTA (6 warps) streams the K/V tiles of one KV head once for a block of
// BM = 128 "packed" query rows: the G query heads that share the KV head times
// their Tq rows (AstrAI commit log, head-packing commit: K/V tiles stream once
// per block instead of once per q head).  Roles:
//   warp 0 lane 0   TMA producer of the Q tile (per segment) and the K ring
//   warp 0 lane 16  TMA producer of the V ring (so a K prefetch never waits
//                   for a V stage to drain)
//   warp 1          TMEM owner; lane 0 issues every tcgen05 MMA:
//                     S = Q K^T   (A, B from shared memory) into TMEM S[g % 2]
//                     O += P V    (A = P from TMEM, B = V from shared memory)
//   warps 2..9      softmax / correction / epilogue: warp w reads TMEM lane
//                     quadrant w % 4 (one packed row per thread) and half
//                     (w - 2) / 4 of every S tile's columns (its exponentials and
//                     its half of O); each reads the whole S row for the row max,
//                     so the two warps of a sub-partition never wait for each
//                     other inside the key loop.  Logical-
//                     length + causal mask by selection, online (m, l) carry with
//                     a lazy rescale of O, P -> bf16 into TMEM P[g % 2], final
//                     O / l (or a normalised partial + lse) to global memory.
//                   With few packed rows (decode) the Q tile is loaded as four
//                   short boxes, one per lane quadrant, so that all four SM
//                   sub-partitions share the softmax work.
// (nvfp4-megamoe-kernel dsv4/kernels/attention commit log: multi-tile commit for
// the online softmax over KV tiles, prefill commits for the TMEM row/lane
// mapping, epilogue commits for TMEM -> registers -> global.)
//
// Work split.  Row-block w = (unit u = (b, kv head), q-tile qt) owns a key
// range of nkv(w) tiles of BN keys.  All tiles of all row-blocks are laid out
// in one flat order and cut into NC equal contiguous spans, one per CTA
// ("stream-K"): every CTA gets the same number of tiles whatever the lengths.
// A row-block finished inside one CTA is written straight to `out`.  One cut by
// span boundaries leaves normalised fp32 partials (O, lse) in per-CTA slots;
// each contributing CTA then takes a ticket on the row-block's counter and the
// last one merges all partials with the LSE combine and writes `out` (AstrAI
// commit log: split-KV scratch commit, and the last-block fold with an atomic
// ticket and fences; kernbench2 benches commit log: associative (m, l, O) merge).
#pragma once
#include <cuda_bf16.h>
#include <cuda.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace gqa {

constexpr int BM = 128;          // packed query rows per tile = TMEM lanes
constexpr int NUM_THREADS = 320; // 10 warps: producers, MMA, 8 softmax warps (2 per lane quadrant)
constexpr int NSOFT = 256;       // softmax threads
constexpr int NSOFT_WARPS = NSOFT / 32;  // arrivals per softmax-side barrier phase (one per warp)
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;
constexpr int kMaxCombinePieces = 512;  // CTA groups of a split (the grid is at most 512 CTAs)  // log2 units: rescale O only when the max grows by > 2^8

// device error codes (same values as gqa_status)
constexpr int DEV_ERR_TIMEOUT = -6;
constexpr int DEV_ERR_KVLEN = -8;
constexpr int DEV_ERR_PAGE = -10;
constexpr int DEV_ERR_SMEM_ALIGN = -11;  // the dynamic shared-memory window was not 1024-byte aligned

// A split row-block (one DSPLIT part of its O columns) whose pieces are all
// written: the stream-K combine kernel merges it.
struct CJob {
    long long pw;   // flat index of the row-block's first tile
    long long tot;  // tiles of the whole problem (the stream-K split)
    int w;          // row-block
    int ntiles;     // its key tiles
    int ho;         // which DSPLIT part of the O columns
    int nc;         // CTA groups of the split
};

struct Params {
    int B, Hq, Hkv, Tq, Tkv, d;
    int G, R, QT, U;      // R = G*Tq rows per unit, QT = ceil(R/BM) q-tiles, U = B*Hkv units
    int RBQ;              // q-tiles per row-block (1, or 2 when two q-tiles share every K/V tile)
    int QW;               // row-blocks per unit = ceil(QT / RBQ)
    long long W;          // row-blocks = U*QW
    int causal;
    int BN;               // keys per tile (the kernel's BN)
    float scale_log2;     // scale * log2(e)  (> 0)
    const int* kv_lens;   // [B] or null
    const float* sink;    // [Hq] or null
    __nv_bfloat16* out;   // [B,Hq,Tq,d]
    float* lse;           // [B,Hq,Tq] or null
    int mode;             // 0: stream-K (direct + slots + in-kernel merge); 1: uniform splits
    int num_splits;       // mode 1
    float* part_o;        // mode 0: [2*NC][BM][d] slots; mode 1: [B,Hq,Tq,S,d]
    float* part_lse;      // mode 0: [2*NC][BM];      mode 1: [B,Hq,Tq,S]
    int* counters;        // mode 0: [W] merge tickets, zero between calls
    int* err;             // device error word
    long long timeout_cycles;
    int q_box_rows;       // rows of one Q TMA box: min(BM, B*Hq*Tq), or rq in the spread layout
    int spread;           // 1: packed row r lives in TMEM lane (r / rq) * 32 + r % rq (R <= 96)
    int rq;               // packed rows per lane quadrant in the spread layout
    int kv_box_rows;      // rows of one K/V TMA box: min(BN, B*Hkv*Tkv)
    CJob* cjobs;          // single-lane kernel, mode 0: [W*DSPLIT] row-blocks for the combine kernel
    int* cjob_count;      // [2]: jobs listed, combine blocks done (zero between calls)
    // paged K/V (two-lane kernel): caches [num_pages, Hkv, page_size, d], page_table
    // [B, max_pages] (logical page -> physical page); page_size 0 = contiguous K/V
    const int* page_table;
    int page_size;
    int max_pages;
    int num_pages;
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

// Key tiles of row-block wq of a unit (its q-tiles wq*RBQ ...), at least one, so
// that a row-block with no visible key is still visited (its one tile is fully
// masked and it writes O = 0).
__host__ __device__ inline int qtile_ntiles(const Params& p, int wq, int n) {
    int ext = 0;
    const int q0 = wq * p.RBQ;
    const int q1 = (q0 + p.RBQ < p.QT) ? q0 + p.RBQ : p.QT;
    for (int qt = q0; qt < q1; ++qt) {
        const int e = qtile_extent(p, qt, n);
        ext = e > ext ? e : ext;
    }
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
    int w;          // row-block
    int t0, t1;     // tile range inside the row-block
    int ntiles;     // nkv(w)
    int n;          // logical length of the row-block's batch
    int kind;       // 0: direct, 1: stream-K slot, 2: uniform split
    int slot;       // slot (kind 1) or split index (kind 2)
    long long pw;   // flat index of the row-block's first tile (kind 0/1)
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
        return static_cast<long long>(p.QW) * (t < 1 ? 1 : t);
    }
    const int lane = threadIdx.x & 31;
    long long acc = 0;
    for (int qt = lane; qt < p.QW; qt += 32) acc += qtile_ntiles(p, qt, n);
    return warp_sum_ll(acc);
}

struct SpanStart {
    long long tot, p0, p1;
    int w, t;
};

// Tiles in one unit of a batch with logical length n (one thread).
__device__ long long unit_tiles_thread(const Params& p, int n) {
    if (!p.causal) {
        int t = (n + p.BN - 1) / p.BN;
        return static_cast<long long>(p.QW) * (t < 1 ? 1 : t);
    }
    long long acc = 0;
    for (int qt = 0; qt < p.QW; ++qt) acc += qtile_ntiles(p, qt, n);
    return acc;
}

// One full warp: total tiles, this CTA's span and the (row-block, tile) where it
// starts.  With per-batch lengths and few row-blocks per unit every lane reads
// its own batches' lengths, so the reads go out together (one memory round trip
// for up to 32 batches), and the batch holding the span's first tile is found
// with a warp scan and a ballot; with many row-blocks per unit (long causal
// prefill) the lanes share each batch's row-blocks instead.
__device__ void plan_span(const Params& p, int c, int NC, SpanStart* out) {
    const int lane = threadIdx.x & 31;
    const bool lane_per_batch = !p.causal || p.QW <= 16;
    long long tot = 0;
    if (p.kv_lens == nullptr) {
        tot = static_cast<long long>(p.U) * unit_tiles_warp(p, p.Tkv);
    } else if (lane_per_batch) {
        long long mine = 0;
        for (int b = lane; b < p.B; b += 32) mine += p.Hkv * unit_tiles_thread(p, load_len(p, b));
        tot = warp_sum_ll(mine);
    } else {
        for (int b = 0; b < p.B; ++b) tot += p.Hkv * unit_tiles_warp(p, load_len(p, b));
    }
    const long long p0 = span_begin(c, tot, NC), p1 = span_begin(c + 1, tot, NC);
    int w = 0, t = 0;
    if (p0 < p1) {
        long long acc = 0;
        int b = 0, n = p.Tkv;
        long long per_unit = 0;
        if (p.kv_lens == nullptr) {
            per_unit = unit_tiles_warp(p, n);
            b = static_cast<int>(p0 / (per_unit * p.Hkv));
            acc = static_cast<long long>(b) * per_unit * p.Hkv;
        } else if (!lane_per_batch) {
            for (b = 0; b < p.B; ++b) {
                n = load_len(p, b);
                per_unit = unit_tiles_warp(p, n);
                if (p0 < acc + per_unit * p.Hkv) break;
                acc += per_unit * p.Hkv;
            }
        } else {
            for (int base = 0; base < p.B; base += 32) {
                const int bb = base + lane;
                const int nb = bb < p.B ? load_len(p, bb) : 0;
                const long long ub = bb < p.B ? unit_tiles_thread(p, nb) : 0;
                const long long cnt = ub * p.Hkv;
                long long inc = cnt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const long long y = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += y;
                }
                const long long chunk_total = __shfl_sync(0xffffffffu, inc, 31);
                if (p0 < acc + chunk_total) {
                    const unsigned hit = __ballot_sync(0xffffffffu, p0 < acc + inc);
                    const int L = __ffs(hit) - 1;
                    b = base + L;
                    n = __shfl_sync(0xffffffffu, nb, L);
                    per_unit = __shfl_sync(0xffffffffu, ub, L);
                    acc += __shfl_sync(0xffffffffu, inc - cnt, L);
                    break;
                }
                acc += chunk_total;
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
            for (int base = 0; base < p.QW; base += 32) {
                const int q = base + lane;
                long long cnt = q < p.QW ? qtile_ntiles(p, q, n) : 0;
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
        w = u * p.QW + qt;
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

// Walks this CTA's segments; every role keeps its own walker and all see the
// same sequence.  Mode 1 has exactly one (possibly empty) segment per CTA.
struct SegWalker {
    int w, t;
    long long remaining, pos;
    bool first, single_done;
    int c;

    __device__ void init(const Params& p, const SpanStart& s, int cta) {
        w = s.w;
        t = s.t;
        remaining = (p.mode == 0) ? s.p1 - s.p0 : 0;
        pos = s.p0;
        first = true;
        single_done = (p.mode == 0);
        c = cta;
    }
    __device__ bool next(const Params& p, Seg& sg) {
        if (!single_done) {  // mode 1: CTA = (row-block, split)
            single_done = true;
            const int S = p.num_splits;
            sg.w = c / S;
            const int s = c % S;
            const int u = sg.w / p.QW, qt = sg.w % p.QW;
            sg.n = load_len(p, u / p.Hkv);
            sg.ntiles = qtile_ntiles(p, qt, sg.n);
            sg.t0 = static_cast<int>((static_cast<long long>(s) * sg.ntiles) / S);
            sg.t1 = static_cast<int>((static_cast<long long>(s + 1) * sg.ntiles) / S);
            sg.kind = 2;
            sg.slot = s;
            sg.pw = 0;
            return true;
        }
        if (remaining <= 0) return false;
        const int u = w / p.QW, qt = w % p.QW;
        const int n = load_len(p, u / p.Hkv);
        const int nt = qtile_ntiles(p, qt, n);
        long long take = nt - t;
        if (take > remaining) take = remaining;
        sg.w = w;
        sg.t0 = t;
        sg.t1 = t + static_cast<int>(take);
        sg.ntiles = nt;
        sg.n = n;
        sg.kind = (t == 0 && sg.t1 == nt) ? 0 : 1;
        sg.slot = first ? 2 * c : 2 * c + 1;
        sg.pw = pos - t;
        pos += take;
        remaining -= take;
        first = false;
        ++w;
        t = 0;
        return true;
    }
};

// ------------------------------------------------------------------ kernel config

// DSPLIT > 1 splits O's columns over DSPLIT CTAs that walk the same key tiles:
// each computes the full S = Q K^T (all D columns of Q and K) but accumulates
// only its DO = D / DSPLIT columns of O, so a 128 x 512 fp32 O never has to fit
// one SM's 512 TMEM columns.
template <int D_, int BN_, int STK_, int STV_, int QBUF_, int DSPLIT_ = 1>
struct FwdCfg {
    static constexpr int D = D_, BN = BN_, STK = STK_, STV = STV_, QBUF = QBUF_, DSPLIT = DSPLIT_;
    static constexpr int DO = D / DSPLIT;               // O columns owned by one CTA
    static_assert(D % 64 == 0 && D <= 512 && DO <= 256 && DO % 64 == 0, "head dim");
    static_assert(BN == 32 || BN == 64 || BN == 128, "key tile");
    static constexpr int HALVES = (BN >= 64) ? 2 : 1;   // softmax column groups per row
    static constexpr int NBOX = D / 64;                 // 64-column swizzle boxes per Q/K row
    static constexpr int VBOX = DO / 64;                // boxes of the V columns this CTA reads
    static constexpr int Q_BOX = BM * 128;              // bytes of one Q box
    static constexpr int Q_BYTES = NBOX * Q_BOX;
    static constexpr int KV_BOX = BN * 128;
    static constexpr int KV_BYTES = NBOX * KV_BOX;      // one K tile
    static constexpr int V_BYTES = VBOX * KV_BOX;       // one V tile (this CTA's columns)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QBUF * Q_BYTES;
    static constexpr int OFF_V = OFF_K + STK * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + STV * V_BYTES;
    // barrier indices
    static constexpr int B_QFULL = 0;
    static constexpr int B_QEMPTY = B_QFULL + QBUF;
    static constexpr int B_KFULL = B_QEMPTY + QBUF;
    static constexpr int B_KEMPTY = B_KFULL + STK;
    static constexpr int B_VFULL = B_KEMPTY + STK;
    static constexpr int B_VEMPTY = B_VFULL + STV;
    static constexpr int B_SFULL = B_VEMPTY + STV;  // [2]
    static constexpr int B_SFREE = B_SFULL + 2;     // [2]
    static constexpr int B_PFULL = B_SFREE + 2;     // [2]
    static constexpr int B_ODONE = B_PFULL + 2;     // [2]
    static constexpr int B_FINAL = B_ODONE + 2;
    static constexpr int B_XSYNC = B_FINAL + 1;     // softmax-group barrier (bounded waits, abort-safe)
    static constexpr int NBAR = B_XSYNC + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int MISC_BYTES = 1664;
    static constexpr int SMEM_USED = OFF_MISC + MISC_BYTES;
    static constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack to align the base to 1024
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    // TMEM columns: O [0, DO), S[2] of BN fp32 columns, P[2] of BN/2 columns (bf16 pairs)
    static constexpr uint32_t TM_O = 0;
    static constexpr uint32_t TM_S = DO;
    static constexpr uint32_t TM_P = DO + 2 * BN;
    static constexpr uint32_t TM_COLS = 512;
    static_assert(DO + 3 * BN <= 512, "TMEM budget");
    static constexpr uint32_t IDESC_S = ptx::umma_idesc_bf16_f32(BM, BN, false, false);
    static constexpr uint32_t IDESC_PV = ptx::umma_idesc_bf16_f32(BM, DO, false, true);
};

struct Misc {
    uint32_t tmem_base;
    volatile int abort;
    volatile int merge_flag;
    int pad;
    SpanStart span;     // 40 bytes
    float red[2][BM];   // per-half row maxima / row sums, by TMEM lane
    float mlse[BM];     // merged lse per packed row (in-kernel merge)
};

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
// Bounded drain used at teardown (no abort short-cut: copies must land).
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t issued, long long limit) {
    if (issued == 0) return;
    const uint32_t par = (issued - 1) & 1;
    const long long t0 = clock64();
    while (!ptx::mbar_try_wait(bar, par) && clock64() - t0 < limit) {
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
    const int u = w / p.QW;
    r.qt = (w % p.QW) * p.RBQ;  // first q-tile of the row-block
    r.b = u / p.Hkv;
    r.g = u % p.Hkv;
    r.q_row0 = (static_cast<long long>(r.b) * p.Hq + static_cast<long long>(r.g) * p.G) * p.Tq +
               static_cast<long long>(r.qt) * BM;
    r.kv_row0 = static_cast<long long>(u) * p.Tkv;
    const int left = p.R - r.qt * BM;
    r.rows_valid = left < BM * p.RBQ ? left : BM * p.RBQ;
    return r;
}

// Slot a contributing CTA wrote for row-block (flat start pw): its first segment
// (2c) unless it is the CTA that holds the row-block's first tile inside a span
// that began earlier (then its last segment, 2c + 1).
__device__ __forceinline__ long long merge_slot(int cc, int c_first, bool c0_first) {
    return (cc == c_first && !c0_first) ? 2ll * cc + 1 : 2ll * cc;
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
    // CTAs come in groups of DSPLIT that walk the same work; ho picks the O columns
    const int ho = static_cast<int>(blockIdx.x) % C::DSPLIT;
    const int cta = static_cast<int>(blockIdx.x) / C::DSPLIT;
    const int NC = static_cast<int>(gridDim.x) / C::DSPLIT;

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
            ptx::mbar_init(bar(C::B_SFREE + i), NSOFT_WARPS);
            ptx::mbar_init(bar(C::B_PFULL + i), NSOFT_WARPS);
            ptx::mbar_init(bar(C::B_ODONE + i), 1);
        }
        ptx::mbar_init(bar(C::B_FINAL), 1);
        ptx::mbar_init(bar(C::B_XSYNC), NSOFT_WARPS);
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
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr(&misc->tmem_base), C::TM_COLS);
        ptx::tmem_relinquish();
    }
    if (p.mode == 0 && warp == 0) plan_span(p, cta, NC, &misc->span);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    // ---------------------------------------------------------------- producers
    if (warp == 0) {
        if (lane == 0) {
            // Q tile per segment + K ring
            const uint64_t pol_q = ptx::policy_evict_last();
            const uint64_t pol_kv = (p.QT == 1) ? ptx::policy_evict_first() : ptx::policy_evict_normal();
            SegWalker wk;
            wk.init(p, misc->span, cta);
            Seg sg;
            int seg_i = 0;
            uint32_t g = 0;
            bool ok = true;
            uint32_t k_issued[C::STK], q_issued[C::QBUF];
            for (int i = 0; i < C::STK; ++i) k_issued[i] = 0;
            for (int i = 0; i < C::QBUF; ++i) q_issued[i] = 0;
            while (ok && wk.next(p, sg)) {
                if (sg.t1 <= sg.t0) continue;  // empty split: nothing to load
                const RB rb = rb_of(p, sg.w);
                const int qb = seg_i % C::QBUF;
                ok = wait_bar(bar(C::B_QEMPTY + qb), ((seg_i / C::QBUF) & 1) ^ 1, misc, p);
                if (!ok) break;
                const int nq = p.spread ? 4 : 1;
                ptx::mbar_arrive_expect_tx(bar(C::B_QFULL + qb), nq * C::NBOX * p.q_box_rows * 128);
                ++q_issued[qb];
                for (int qq = 0; qq < nq; ++qq)
                    for (int bx = 0; bx < C::NBOX; ++bx)
                        ptx::tma_load_2d(sbase + C::OFF_Q + qb * C::Q_BYTES + bx * C::Q_BOX + qq * 32 * 128, &tm_q,
                                         bx * 64, static_cast<int>(rb.q_row0) + qq * p.rq, bar(C::B_QFULL + qb),
                                         pol_q);
                for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                    const int st = g % C::STK;
                    ok = wait_bar(bar(C::B_KEMPTY + st), ((g / C::STK) & 1) ^ 1, misc, p);
                    if (!ok) break;
                    const int y = static_cast<int>(rb.kv_row0 + static_cast<long long>(t) * C::BN);
                    ptx::mbar_arrive_expect_tx(bar(C::B_KFULL + st), C::NBOX * p.kv_box_rows * 128);
                    ++k_issued[st];
                    for (int bx = 0; bx < C::NBOX; ++bx)
                        ptx::tma_load_2d(sbase + C::OFF_K + st * C::KV_BYTES + bx * C::KV_BOX, &tm_k, bx * 64, y,
                                         bar(C::B_KFULL + st), pol_kv);
                }
                ++seg_i;
            }
            // never leave the CTA with copies in flight
            for (int i = 0; i < C::STK; ++i) drain_bar(bar(C::B_KFULL + i), k_issued[i], p.timeout_cycles);
            for (int i = 0; i < C::QBUF; ++i) drain_bar(bar(C::B_QFULL + i), q_issued[i], p.timeout_cycles);
        } else if (lane == 16) {
            // V ring
            const uint64_t pol_kv = (p.QT == 1) ? ptx::policy_evict_first() : ptx::policy_evict_normal();
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
                    ok = wait_bar(bar(C::B_VEMPTY + st), ((g / C::STV) & 1) ^ 1, misc, p);
                    if (!ok) break;
                    const int y = static_cast<int>(rb.kv_row0 + static_cast<long long>(t) * C::BN);
                    ptx::mbar_arrive_expect_tx(bar(C::B_VFULL + st), C::VBOX * p.kv_box_rows * 128);
                    ++v_issued[st];
                    for (int bx = 0; bx < C::VBOX; ++bx)
                        ptx::tma_load_2d(sbase + C::OFF_V + st * C::V_BYTES + bx * C::KV_BOX, &tm_v,
                                         ho * C::DO + bx * 64, y, bar(C::B_VFULL + st), pol_kv);
                }
            }
            for (int i = 0; i < C::STV; ++i) drain_bar(bar(C::B_VFULL + i), v_issued[i], p.timeout_cycles);
        }
    }
    // ---------------------------------------------------------------- MMA issuer
    else if (warp == 1) {
        if (lane == 0) {
            SegWalker wk;
            wk.init(p, misc->span, cta);
            Seg sg;
            int seg_i = 0;
            uint32_t g = 0;
            bool ok = true;
            bool have_prev = false;   // a PV is pending for tile g-1
            bool prev_first = false;  // ... and it is the first tile of its segment
            const uint32_t tm_o = tmem + C::TM_O;

            auto issue_pv = [&](uint32_t gp, bool first_of_seg) -> bool {
                const int pb = gp & 1;
                if (!wait_bar(bar(C::B_PFULL + pb), (gp >> 1) & 1, misc, p)) return false;
                const int st = gp % C::STV;
                if (!wait_bar(bar(C::B_VFULL + st), (gp / C::STV) & 1, misc, p)) return false;
                ptx::tc_fence_after();
                const uint32_t vbase = sbase + C::OFF_V + st * C::V_BYTES;
                const uint32_t tm_p = tmem + C::TM_P + pb * (C::BN / 2);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    const uint64_t bd = ptx::umma_desc_sw128(vbase + kk * 2048, C::KV_BOX, 1024);
                    ptx::umma_bf16_ts(tm_o, tm_p + kk * 8, bd, C::IDESC_PV, (kk > 0 || !first_of_seg) ? 1u : 0u);
                }
                ptx::umma_commit(bar(C::B_ODONE + pb));
                ptx::umma_commit(bar(C::B_VEMPTY + st));
                return true;
            };

            while (ok && wk.next(p, sg)) {
                if (sg.t1 <= sg.t0) continue;
                const int qb = seg_i % C::QBUF;
                ok = wait_bar(bar(C::B_QFULL + qb), (seg_i / C::QBUF) & 1, misc, p);
                if (!ok) break;
                const uint32_t qbase = sbase + C::OFF_Q + qb * C::Q_BYTES;
                for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                    const int st = g % C::STK;
                    const int sb = g & 1;
                    ok = wait_bar(bar(C::B_KFULL + st), (g / C::STK) & 1, misc, p);
                    if (!ok) break;
                    if (g >= 2) {
                        ok = wait_bar(bar(C::B_SFREE + sb), ((g >> 1) - 1) & 1, misc, p);
                        if (!ok) break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t kbase = sbase + C::OFF_K + st * C::KV_BYTES;
                    const uint32_t tm_s = tmem + C::TM_S + sb * C::BN;
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
            // every MMA must retire before TMEM is released
            ptx::umma_commit(bar(C::B_FINAL));
            drain_bar(bar(C::B_FINAL), 1, p.timeout_cycles);
        }
    }
    // ---------------------------------------------------------------- softmax / epilogue
    else {
        const int quad = warp & 3;             // TMEM lane quadrant this warp may access
        const int half = (warp - 2) >> 2;      // which half of the key columns / O columns
        const int lrow = quad * 32 + lane;     // TMEM lane = row of the MMA tile
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        constexpr int HB = C::BN / C::HALVES;  // key columns per half
        constexpr int HD = C::DO / C::HALVES;  // O columns per half
        const uint32_t tm_o = tmem + lane_off + C::TM_O + half * HD;
        const int stid = threadIdx.x - 64;     // 0..255 among the softmax threads
        // Barrier over the 256 softmax threads on an mbarrier with a bounded wait, so
        // that an abort elsewhere can never leave threads parked at it.
        uint32_t xph = 0;
        auto xsync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(C::B_XSYNC));
            const bool r = wait_bar(bar(C::B_XSYNC), xph & 1, misc, p);
            ++xph;
            return __all_sync(0xffffffffu, r);
        };
        SegWalker wk;
        wk.init(p, misc->span, cta);
        Seg sg;
        uint32_t g = 0;
        bool ok = true;

        while (ok && wk.next(p, sg)) {
            const RB rb = rb_of(p, sg.w);
            // packed row held by this thread
            int rloc;                           // row inside the q-tile
            bool valid, active;
            if (p.spread) {
                rloc = quad * p.rq + lane;
                valid = lane < p.rq && rloc < rb.rows_valid;
                active = quad * p.rq < rb.rows_valid;
            } else {
                rloc = lrow;
                valid = lrow < rb.rows_valid;
                active = quad * 32 < rb.rows_valid;
            }
            // with a single column group the second group's warps only keep the barrier counts
            active = active && half < C::HALVES;
            const int rp = rb.qt * BM + rloc;   // packed row inside the unit
            const int hl = valid ? rp / p.Tq : 0;
            const int i = valid ? rp % p.Tq : 0;
            int limit = p.causal ? (sg.n - p.Tq + i) : (sg.n - 1);
            if (limit > sg.n - 1) limit = sg.n - 1;
            if (!valid) limit = -1;
            const int h = rb.g * p.G + hl;

            float m_ref = -INFINITY;  // log2-domain running max the P values are taken against
            float l_sum = 0.f;        // this half's running sum

            for (int t = sg.t0; t < sg.t1; ++t, ++g) {
                const int sb = g & 1;
                ok = wait_bar(bar(C::B_SFULL + sb), (g >> 1) & 1, misc, p);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ptx::tc_fence_after();
                float s[HB];
                float mx = -INFINITY;
                if (active) {
                    const uint32_t tm_s = tmem + lane_off + C::TM_S + sb * C::BN;
                    // own half: kept for the exponentials
#pragma unroll
                    for (int c = 0; c < HB / 32; ++c) {
                        uint32_t r[32];
                        ptx::tmem_ld32(tm_s + half * HB + c * 32, r);
#pragma unroll
                        for (int j = 0; j < 32; ++j) s[c * 32 + j] = __uint_as_float(r[j]);
                    }
                    ptx::tmem_wait_ld();
                    // mask by selection (never by adding -inf: NaN + -inf stays NaN)
                    const int lim_all = limit - t * C::BN;      // last visible column of the tile
                    const bool full = __all_sync(0xffffffffu, lim_all >= C::BN - 1);
                    const int lim = lim_all - half * HB;
                    if (!full) {
#pragma unroll
                        for (int c = 0; c < HB; ++c) s[c] = (c <= lim) ? s[c] : -INFINITY;
                    }
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < HB; c += 4) {
                        m4[0] = fmaxf(m4[0], s[c]);
                        m4[1] = fmaxf(m4[1], s[c + 1]);
                        m4[2] = fmaxf(m4[2], s[c + 2]);
                        m4[3] = fmaxf(m4[3], s[c + 3]);
                    }
                    // other half: only its maximum is needed
                    const int olim = lim_all - (half ^ 1) * HB;
#pragma unroll
                    for (int c = 0; c < (C::HALVES == 2 ? HB / 32 : 0); ++c) {
                        uint32_t r[32];
                        ptx::tmem_ld32(tm_s + (half ^ 1) * HB + c * 32, r);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float x = __uint_as_float(r[j + e]);
                                m4[e] = fmaxf(m4[e], (full || c * 32 + j + e <= olim) ? x : -INFINITY);
                            }
                        }
                    }
                    mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::B_SFREE + sb));

                const bool first = (t == sg.t0);
                float alpha = 1.f;
                const float mt = mx * p.scale_log2;  // -inf stays -inf (scale > 0)
                if (first) {
                    m_ref = mt;
                } else if (mt > m_ref + RESCALE_THRESHOLD) {
                    alpha = ptx::ex2(m_ref - mt);
                    m_ref = mt;
                }
                // P buffer g%2 was last read by PV_{g-2}
                const int pb = g & 1;
                if (g >= 2) {
                    ok = wait_bar(bar(C::B_ODONE + pb), ((g >> 1) - 1) & 1, misc, p);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    ptx::tc_fence_after();
                }
                if (active) {
                    const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
                    const uint32_t tm_p = tmem + lane_off + C::TM_P + pb * (C::BN / 2) + half * (HB / 2);
                    float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int c = 0; c < HB / 32; ++c) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float a = ptx::ex2(fmaf(s[c * 32 + 2 * j], p.scale_log2, neg_m));
                            const float b = ptx::ex2(fmaf(s[c * 32 + 2 * j + 1], p.scale_log2, neg_m));
                            rs4[(2 * j) & 3] += a;
                            rs4[(2 * j + 1) & 3] += b;
                            pk[j] = pack_bf16x2(a, b);
                        }
                        ptx::tmem_st16(tm_p + c * 16, pk);
                    }
                    l_sum = l_sum * alpha + ((rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
                    // lazy rescale of this half of O: only when some row's max grew by more than 2^8
                    if (!first && __any_sync(0xffffffffu, alpha != 1.f)) {
                        bool okw = wait_bar(bar(C::B_ODONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, misc, p);
                        okw = __all_sync(0xffffffffu, okw);
                        if (!okw) {
                            ok = false;
                        } else {
                            ptx::tc_fence_after();
#pragma unroll 1
                            for (int c = 0; c < HD / 32; ++c) {
                                uint32_t r[32];
                                ptx::tmem_ld32(tm_o + c * 32, r);
                                ptx::tmem_wait_ld();
#pragma unroll
                                for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
                                ptx::tmem_st32(tm_o + c * 32, r);
                            }
                        }
                    }
                    ptx::tmem_wait_st();
                }
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                // padded key rows of the V tile must reach the MMA as zeros (0 * NaN = NaN)
                if ((t + 1) * C::BN > sg.n) {
                    const int st = g % C::STV;
                    ok = wait_bar(bar(C::B_VFULL + st), (g / C::STV) & 1, misc, p);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    int z0 = sg.n - t * C::BN;
                    z0 = z0 < 0 ? 0 : z0;
                    uint8_t* vt = smem + C::OFF_V + st * C::V_BYTES;
                    const int chunks = (C::BN - z0) * C::VBOX * 8;  // 16-byte chunks
                    for (int q = stid; q < chunks; q += NSOFT) {
                        const int r = z0 + q / (C::VBOX * 8);
                        const int rem = q % (C::VBOX * 8);
                        *reinterpret_cast<uint4*>(vt + (rem >> 3) * C::KV_BOX + r * 128 + (rem & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::B_PFULL + pb));
            }
            if (!ok) break;

            // ------------------------------------------------ segment epilogue
            const bool nonempty = sg.t1 > sg.t0;
            misc->red[half][lrow] = l_sum;
            if (!xsync()) { ok = false; break; }
            const float l_tot = l_sum + misc->red[half ^ 1][lrow];
            if (nonempty) {
                const uint32_t gl = g - 1;
                ok = wait_bar(bar(C::B_ODONE + (gl & 1)), (gl >> 1) & 1, misc, p);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ptx::tc_fence_after();
            }
            float o_scale = 0.f, lse_v = -INFINITY;
            if (nonempty) {
                if (sg.kind == 0) {
                    const float sk = (p.sink != nullptr && valid) ? __ldg(p.sink + h) * LOG2E : -INFINITY;
                    const float M = fmaxf(m_ref, sk);
                    if (M != -INFINITY) {
                        const float a = ptx::ex2(m_ref - M);
                        const float lt = l_tot * a + ptx::ex2(sk - M);
                        o_scale = a / lt;
                        lse_v = (M + __log2f(lt)) * LN2;
                    }
                } else if (l_tot > 0.f) {
                    o_scale = 1.f / l_tot;
                    lse_v = (m_ref + __log2f(l_tot)) * LN2;
                }
            }
            const long long fr = rb.q_row0 + rloc;  // flat row (b*Hq + h)*Tq + i when valid
            if (sg.kind == 0) {
                __nv_bfloat16* dst = p.out + fr * C::D + ho * C::DO + half * HD;
                if (active) {
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t r[32];
                        ptx::tmem_ld32(tm_o + c * 32, r);
                        ptx::tmem_wait_ld();
                        if (valid) {
                            uint32_t pk[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                pk[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * o_scale,
                                                    __uint_as_float(r[2 * j + 1]) * o_scale);
                            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                d4[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                        }
                    }
                }
                if (valid && half == 0 && ho == 0 && p.lse != nullptr) p.lse[fr] = lse_v;
            } else {
                // stream-K slots hold [BM rows][DO columns] per CTA of a DSPLIT group
                float* dst;
                float* dl;
                if (sg.kind == 1) {
                    const long long slot = static_cast<long long>(sg.slot) * C::DSPLIT + ho;
                    dst = p.part_o + (slot * BM + rloc) * C::DO + half * HD;
                    dl = p.part_lse + slot * BM + rloc;
                } else {
                    dst = p.part_o + (fr * p.num_splits + sg.slot) * C::D + ho * C::DO + half * HD;
                    dl = p.part_lse + fr * p.num_splits + sg.slot;
                }
                if (active) {
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t r[32];
                        if (nonempty) {
                            ptx::tmem_ld32(tm_o + c * 32, r);
                            ptx::tmem_wait_ld();
                        }
                        if (valid) {
                            float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                                if (nonempty)
                                    v4 = make_float4(__uint_as_float(r[4 * j]) * o_scale,
                                                     __uint_as_float(r[4 * j + 1]) * o_scale,
                                                     __uint_as_float(r[4 * j + 2]) * o_scale,
                                                     __uint_as_float(r[4 * j + 3]) * o_scale);
                                __stcg(d4 + j, v4);
                            }
                        }
                    }
                }
                if (valid && half == 0 && (sg.kind == 1 || ho == 0)) __stcg(dl, lse_v);

                if (sg.kind == 1) {
                    // ---- ticket: the CTA that completes the row-block's pieces lists it for the
                    // stream-K combine kernel, which merges every listed row-block across all SMs
                    // (it runs after this kernel, so the partial rows need no fence here)
                    const long long tot = misc->span.tot;
                    const int c_first = cta_of(sg.pw, tot, NC);
                    const int c_last = cta_of(sg.pw + sg.ntiles - 1, tot, NC);
                    if (!xsync()) { ok = false; break; }
                    if (stid == 0) {
                        int ncontrib = 0;
                        for (int cc = c_first; cc <= c_last; ++cc)
                            ncontrib += span_begin(cc, tot, NC) < span_begin(cc + 1, tot, NC);
                        const long long ctr = static_cast<long long>(sg.w) * C::DSPLIT + ho;
                        const int old = atomicAdd(p.counters + ctr, 1);
                        if (old == ncontrib - 1) {
                            p.counters[ctr] = 0;  // ready for the next call
                            CJob jb;
                            jb.pw = sg.pw;
                            jb.tot = tot;
                            jb.w = sg.w;
                            jb.ntiles = sg.ntiles;
                            jb.ho = ho;
                            jb.nc = NC;
                            p.cjobs[atomicAdd(p.cjob_count, 1)] = jb;
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            // misc->red / mlse / merge_flag are reused by the next segment
            if (!xsync()) { ok = false; break; }
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

// ------------------------------------------------------------------ public combine kernel

// Uniform combine (public entry): one warp per row, S partials laid out [rows, S, d].
// Stream-K combine (single-lane kernel, mode 0): merges the row-blocks the main
// kernel listed, each from its pieces' partial (O, lse) in the slots 2c / 2c + 1 of
// the CTA groups c that hold a piece, into O (bf16) and lse:
//   lse = log(e^sink + sum_k e^lse_k),  O = sum_k e^(lse_k - lse) O_k.
// A block takes 8 rows of one listed row-block at a time (grid-stride over all of
// them): one warp per row finds its lse and the pieces' weights, then every
// thread sums 8 columns of a row over the pieces, four pieces' loads at a time.
// The last block to finish leaves the job counter at zero for the next call.
constexpr int kCombRows = 8;
__global__ void __launch_bounds__(256)
gqa_combine_streamk_kernel(const Params p, int dsplit, int rw) {
    __shared__ int slot_s[kMaxCombinePieces];
    __shared__ float wgt_s[kCombRows][kMaxCombinePieces];
    __shared__ int npieces_s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int njobs = *reinterpret_cast<volatile int*>(p.cjob_count);
    const int DO = p.d / dsplit;
    const int chunks = (rw + kCombRows - 1) / kCombRows;
    const long long units = static_cast<long long>(njobs) * chunks;
    for (long long u = blockIdx.x; u < units; u += gridDim.x) {
        const CJob jb = p.cjobs[u / chunks];
        const int r0 = static_cast<int>(u % chunks) * kCombRows;
        const RB rb = rb_of(p, jb.w);
        const int nrows = min(kCombRows, rb.rows_valid - r0);
        if (nrows <= 0) continue;
        const int c_first = cta_of(jb.pw, jb.tot, jb.nc);
        const int c_last = cta_of(jb.pw + jb.ntiles - 1, jb.tot, jb.nc);
        const bool c0_first = span_begin(c_first, jb.tot, jb.nc) == jb.pw;
        if (warp == 0) {
            int nm = 0;
            for (int base = c_first; base <= c_last; base += 32) {
                const int cc = base + lane;
                const bool has = cc <= c_last && span_begin(cc, jb.tot, jb.nc) < span_begin(cc + 1, jb.tot, jb.nc);
                const unsigned m = __ballot_sync(0xffffffffu, has);
                const int k = nm + __popc(m & ((1u << lane) - 1u));
                if (has && k < kMaxCombinePieces)
                    slot_s[k] = static_cast<int>(merge_slot(cc, c_first, c0_first) * dsplit + jb.ho);
                nm += __popc(m);
            }
            if (lane == 0) npieces_s = nm < kMaxCombinePieces ? nm : kMaxCombinePieces;
        }
        __syncthreads();
        const int np = npieces_s;
        // lse and the pieces' weights of each row: one warp per row
        if (warp < nrows) {
            const int r = r0 + warp;
            const int hr = rb.g * p.G + (rb.qt * BM + r) / p.Tq;
            const float sk = (p.sink != nullptr) ? __ldg(p.sink + hr) : -INFINITY;
            float mx = sk;
            for (int k = lane; k < np; k += 32) mx = fmaxf(mx, __ldcg(p.part_lse + static_cast<long long>(slot_s[k]) * rw + r));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float z = 0.f;
            if (mx != -INFINITY) {
                for (int k = lane; k < np; k += 32) z += __expf(__ldcg(p.part_lse + static_cast<long long>(slot_s[k]) * rw + r) - mx);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
                if (sk != -INFINITY) z += __expf(sk - mx);
            }
            const float lt = (mx != -INFINITY && z > 0.f) ? mx + __logf(z) : -INFINITY;
            for (int k = lane; k < np; k += 32)
                wgt_s[warp][k] = (lt != -INFINITY) ? __expf(__ldcg(p.part_lse + static_cast<long long>(slot_s[k]) * rw + r) - lt) : 0.f;
            if (lane == 0 && p.lse != nullptr && jb.ho == 0) p.lse[rb.q_row0 + r] = lt;
        }
        __syncthreads();
        // O: 8 columns per item
        const int C8 = DO / 8;
        for (int it = threadIdx.x; it < nrows * C8; it += blockDim.x) {
            const int rr = it / C8, c8 = it % C8;
            const int r = r0 + rr;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int k0 = 0; k0 < np; k0 += 4) {
                float4 xa[4], xb[4];
                float wk[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (k0 + j < np) {
                        const float4* src = reinterpret_cast<const float4*>(
                            p.part_o + (static_cast<long long>(slot_s[k0 + j]) * rw + r) * DO + 8 * c8);
                        xa[j] = __ldcg(src);
                        xb[j] = __ldcg(src + 1);
                        wk[j] = wgt_s[rr][k0 + j];
                    } else {
                        xa[j] = xb[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                        wk[j] = 0.f;
                    }
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[0] += wk[j] * xa[j].x; acc[1] += wk[j] * xa[j].y; acc[2] += wk[j] * xa[j].z; acc[3] += wk[j] * xa[j].w;
                    acc[4] += wk[j] * xb[j].x; acc[5] += wk[j] * xb[j].y; acc[6] += wk[j] * xb[j].z; acc[7] += wk[j] * xb[j].w;
                }
            }
            *reinterpret_cast<uint4*>(p.out + (rb.q_row0 + r) * p.d + jb.ho * DO + 8 * c8) =
                make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                           pack_bf16x2(acc[6], acc[7]));
        }
        __syncthreads();  // slot_s / wgt_s are rewritten by the next unit
    }
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.cjob_count + 1, 1) == static_cast<int>(gridDim.x) - 1) {
            p.cjob_count[0] = 0;
            p.cjob_count[1] = 0;
        }
    }
}

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

// ------------------------------------------------------------------ key shards
// Sequence parallelism over a key-sharded K/V cache: the rank that holds keys
// [key_offset, key_offset + capacity) of every sequence sees min(n, ...) of them.
__global__ void gqa_shard_lengths_kernel(const int* __restrict__ kv_lens, int B, int key_offset, int capacity,
                                         int* __restrict__ shard_lens) {
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) {
        const long long n = static_cast<long long>(kv_lens[b]) - key_offset;
        shard_lens[b] = static_cast<int>(n < 0 ? 0 : (n > capacity ? capacity : n));
    }
}

// LSE merge of per-shard results: shard s holds, for every row, its output over
// the shard's keys (bf16, normalised) and that sum's lse (-inf: no visible key);
// shard s of the outputs starts s * o_stride elements after the first, of the
// lse s * l_stride elements after.  One warp per output row; the sink enters
// once, here.
__global__ void __launch_bounds__(256)
gqa_combine_shards_kernel(const __nv_bfloat16* __restrict__ o_sh, long long o_stride, const float* __restrict__ l_sh,
                          long long l_stride, int S, const float* __restrict__ sink, __nv_bfloat16* __restrict__ out,
                          float* __restrict__ lse, long long rows, int Hq, int Tq, int d) {
    extern __shared__ float wsh[];  // [8 warps][S]
    const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* wts = wsh + wib * S;
    const long long nwarps = static_cast<long long>(gridDim.x) * 8;
    for (long long row = static_cast<long long>(blockIdx.x) * 8 + wib; row < rows; row += nwarps) {
        const int h = static_cast<int>((row / Tq) % Hq);
        const float sk = (sink != nullptr) ? sink[h] : -INFINITY;
        float L = sk;
        for (int s = lane; s < S; s += 32) L = fmaxf(L, l_sh[s * l_stride + row]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L = fmaxf(L, __shfl_xor_sync(0xffffffffu, L, o));
        float lt = -INFINITY;
        if (L != -INFINITY) {
            float z = 0.f;
            for (int s = lane; s < S; s += 32) z += __expf(l_sh[s * l_stride + row] - L);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            if (sink != nullptr) z += __expf(sk - L);
            lt = L + __logf(z);
        }
        for (int s = lane; s < S; s += 32) wts[s] = (lt == -INFINITY) ? 0.f : __expf(l_sh[s * l_stride + row] - lt);
        __syncwarp();
        for (int c4 = lane; c4 < d / 4; c4 += 32) {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            for (int s = 0; s < S; ++s) {
                const float wgt = wts[s];
                if (wgt == 0.f) continue;
                const uint2 raw = *reinterpret_cast<const uint2*>(o_sh + s * o_stride + row * d + 4 * c4);
                const __nv_bfloat162 x01 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
                const __nv_bfloat162 x23 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
                a0 += wgt * __low2float(x01);
                a1 += wgt * __high2float(x01);
                a2 += wgt * __low2float(x23);
                a3 += wgt * __high2float(x23);
            }
            *reinterpret_cast<uint2*>(out + row * d + 4 * c4) = make_uint2(pack_bf16x2(a0, a1), pack_bf16x2(a2, a3));
        }
        if (lane == 0 && lse != nullptr) lse[row] = lt;
        __syncwarp();
    }
}

}  // namespace gqa

static_assert(sizeof(gqa::Misc) <= 1664, "misc block");
