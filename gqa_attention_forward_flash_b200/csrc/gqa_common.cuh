// gqa_common.cuh -- pieces shared by the sm_100a GQA attention kernels: the
// kernel parameters, the stream-K work split (plan of each CTA's span, the walk
// over its segments), bounded mbarrier waits, row-block geometry, and the small
// combine kernels (the public uniform-split LSE combine and the key-shard merge).
//
// Work split ("stream-K").  Row-block w = (unit u = (b, kv head), q-tile qt) owns
// a key range of nkv(w) tiles of BN keys.  All tiles of all row-blocks are laid
// out in one flat order and cut into NC equal contiguous spans, one per CTA (or
// CTA group): every CTA gets the same number of tiles whatever the lengths.  A
// row-block finished inside one CTA is written straight to `out`; one cut by
// span boundaries leaves normalised fp32 partials (O, lse) in per-CTA slots,
// merged with the LSE combine (AstrAI commit log: split-KV scratch commit, and
// the last-block fold with an atomic ticket and fences; kernbench2 benches commit
// log: associative (m, l, O) merge).
#pragma once
#include <cuda_bf16.h>
#include <cuda.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace gqa {

constexpr int BM = 128;          // packed query rows per tile = TMEM lanes
constexpr int kMaxGrid = 512;    // CTAs (or CTA groups) of a stream-K launch at most
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

// device error codes (same values as gqa_status)
constexpr int DEV_ERR_TIMEOUT = -6;
constexpr int DEV_ERR_KVLEN = -8;
constexpr int DEV_ERR_PAGE = -10;
constexpr int DEV_ERR_SMEM_ALIGN = -11;  // the dynamic shared-memory window was not 1024-byte aligned

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
    float* part_o;        // mode 0: 2 slots per CTA of [BM*RBQ rows][d] (layout per kernel); mode 1: [B,Hq,Tq,S,d]
    float* part_lse;      // mode 0: 2 slots per CTA of [BM*RBQ];                         mode 1: [B,Hq,Tq,S]
    int* counters;        // mode 0: merge counters per row-block, zero between calls
    int* err;             // device error word
    long long timeout_cycles;
    int q_box_rows;       // rows of one Q TMA box: min(BM, B*Hq*Tq), or rq in the spread layout
    int spread;           // 1: packed row r lives in TMEM lane (r / rq) * 32 + r % rq (R <= 96)
    int rq;               // packed rows per lane quadrant in the spread layout
    int kv_box_rows;      // rows of one K/V TMA box: min(BN, B*Hkv*Tkv)
    // paged K/V (two-lane kernel): caches [num_pages, Hkv, page_size, d], page_table
    // [B, max_pages] (logical page -> physical page); page_size 0 = contiguous K/V
    const int* page_table;
    int page_size;
    int max_pages;
    int num_pages;
    // FP8 K/V (swap-AB decode kernel): K/V are E4M3 bytes; k_scale is folded into
    // scale_log2, v_scale multiplies the normalised output (1 otherwise)
    int kv_fp8;
    float v_scale;
    // cost-weighted spans (swap-AB decode kernel): every row-block start counts as
    // seg_w extra tiles when the flat order is cut into equal spans, so that a CTA
    // whose span crosses more row-blocks (more epilogues, merges, segment
    // switches) gets fewer tiles; 0 = equal spans of tiles
    int seg_w;
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

// Cost-weighted spans (row-blocks of one q-tile: QW == 1).  Unit u = (b, g) has
// nt(b) tiles and counts as E + nt(b) in weighted positions (E = p.seg_w): its
// weighted extent [Y(u), Y(u) + E + nt(b)) with Y(u) = T(u) + u*E, T(u) its first
// flat tile.  CTA c owns the weighted interval [c*tot_w/NC, (c+1)*tot_w/NC); a
// weighted position y inside unit u maps to the flat tile T(u) + max(0, y - Y(u) - E)
// (the first E positions of a unit carry its start-up cost and no tile).
//
// yb[b] (b = 0..B) is the weighted start of batch b's first unit, built by one
// warp; from it, one thread maps boundary k to the flat start of CTA k's span
// (and, for the CTA's own start, its row-block and tile).
constexpr int kMaxWeightedB = 1024;  // batches the weighted plan keeps in its table

__device__ int weighted_bound(const Params& p, const int* yb, int NC, int k, int* w_out, int* t_out) {
    const long long E = p.seg_w;
    const long long tot_w = yb[p.B];
    const long long tot = tot_w - static_cast<long long>(p.B) * p.Hkv * E;
    const long long y = (static_cast<long long>(k) * tot_w) / NC;
    if (y >= tot_w) {
        *w_out = 0;
        *t_out = 0;
        return static_cast<int>(tot);
    }
    int lo = 0, hi = p.B;  // yb[lo] <= y < yb[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (yb[mid] <= y) lo = mid;
        else hi = mid;
    }
    const int per_unit = (yb[lo + 1] - yb[lo]) / p.Hkv;  // E + nt(b)
    const int n = per_unit - static_cast<int>(E);
    const int off = static_cast<int>(y - yb[lo]);
    const int g = off / per_unit, r = off - g * per_unit;
    const int t = r > E ? r - static_cast<int>(E) : 0;
    *w_out = lo * p.Hkv + g;
    *t_out = t;
    return static_cast<int>(yb[lo] - static_cast<long long>(lo) * p.Hkv * E) + g * n + t;
}

// One full warp: the batch table yb[0..B] and this CTA's SpanStart.
__device__ void plan_span_weighted(const Params& p, int c, int NC, SpanStart* out, int* yb, int* lens = nullptr) {
    const int lane = threadIdx.x & 31;
    const int E = p.seg_w;
    int acc = 0;
    for (int base = 0; base < p.B; base += 32) {
        const int bb = base + lane;
        const int n = bb < p.B ? load_len(p, bb) : 0;
        if (lens != nullptr && bb < p.B) lens[bb] = n;
        const int lw = bb < p.B ? p.Hkv * (qtile_ntiles(p, 0, n) + E) : 0;
        int inc = lw;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        if (bb < p.B) yb[bb] = acc + inc - lw;
        acc += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) yb[p.B] = acc;
    __syncwarp();
    // lanes 0 and 1: the two boundaries of this CTA's span
    int w = 0, t = 0, f = 0;
    if (lane < 2) f = weighted_bound(p, yb, NC, c + lane, &w, &t);
    const int f1 = __shfl_sync(0xffffffffu, f, 1);
    if (lane == 0) {
        out->tot = acc - static_cast<long long>(p.B) * p.Hkv * E;
        out->p0 = f;
        out->p1 = f1;
        out->w = w;
        out->t = t;
    }
}

// One full warp: bounds[k] = flat start of CTA k's span, k = 0..NC.
__device__ void fill_span_bounds(const Params& p, const int* yb, int NC, int* bounds) {
    const int lane = threadIdx.x & 31;
    for (int k = lane; k <= NC; k += 32) {
        int w, t;
        bounds[k] = weighted_bound(p, yb, NC, k, &w, &t);
    }
    __syncwarp();
}

// Owner of flat tile x under a bounds table: the last c with bounds[c] <= x.
__device__ __forceinline__ int cta_of_table(const int* bounds, int NC, long long x) {
    int lo = 0, hi = NC;  // bounds[lo] <= x < bounds[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (bounds[mid] <= x) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Walks this CTA's segments; every role keeps its own walker and all see the
// same sequence.  Mode 1 has exactly one (possibly empty) segment per CTA.
struct SegWalker {
    int w, t;
    long long remaining, pos;
    bool first, single_done;
    int c;
    const int* lens;  // the batches' logical lengths in shared memory, or null (read them from global)

    __device__ void init(const Params& p, const SpanStart& s, int cta, const int* len_table = nullptr) {
        lens = len_table;
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
        const int n = lens ? lens[u / p.Hkv] : load_len(p, u / p.Hkv);
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

// The head of every kernel's shared-memory control block (each kernel's own block
// starts with these fields): the bounded waits read the CTA abort flag here.
struct Misc {
    uint32_t tmem_base;
    volatile int abort;
    volatile int merge_flag;
    int pad;
    SpanStart span;
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

// NaN propagation through the row statistics: a row that met a NaN score or
// value has a NaN row sum, and its output and log-sum-exp must come out NaN
// (as IEEE arithmetic on the definition gives), so the maxima below keep NaN
// (fmaxf would drop it) and a NaN sum takes the branch of a positive one.
__device__ __forceinline__ float fmax_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ bool pos_or_nan(float x) { return !(x <= 0.f); }

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

// ------------------------------------------------------------------ public combine kernel

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
        for (int s = lane; s < S; s += 32) L = fmax_nan(L, lse_part[row * S + s]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L = fmax_nan(L, __shfl_xor_sync(0xffffffffu, L, o));
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
        for (int s = lane; s < S; s += 32) L = fmax_nan(L, l_sh[s * l_stride + row]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L = fmax_nan(L, __shfl_xor_sync(0xffffffffu, L, o));
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
