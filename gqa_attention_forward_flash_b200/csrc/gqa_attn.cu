// gqa_attn.cu -- host side of the C ABI declared in include/gqa_attn.h:
// argument validation, kernel choice per head dim, TMA descriptors, the
// per-device scratch for split partials, launches.
//
// Validation follows the rules the AstrAI commit log lists for its attention
// bindings (q-head / kv-head divisibility, head-dim contiguity, split-KV scratch
// layout) and its rule not to swallow cudaFuncSetAttribute failures.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gqa_attn.h"
#include "gqa_dec_kernel.cuh"
#include "gqa_wide_kernel.cuh"

namespace gqa {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxCtas = 512;  // the stream-K combine keeps its slot list in 512 entries

struct DeviceState {
    bool init = false;
    int sm_count = 0;
    int cc_major = 0, cc_minor = 0;
    long long clock_khz = 0;
    int* err = nullptr;          // device error word
    void* scratch = nullptr;     // stream-K partial slots (O, lse)
    size_t scratch_bytes = 0;
    int* counters = nullptr;     // per-row-block merge tickets, all zero between calls
    long long counters_len = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// Optional per-launch timing (gqa_profile_*): events recorded on the launch
// stream right before and right after the one kernel of each
// gqa_attention_fwd call, read back by gqa_profile_take.
constexpr int kProfCap = 4096;
struct Prof {
    bool on = false;
    int dev = -1;
    int n = 0;
    cudaEvent_t ev[kProfCap][2];
    bool created = false;
};
Prof g_prof;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_state(DeviceState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
    DeviceState& s = g_dev[dev];
    if (!s.init) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return GQA_ERR_CUDA;
        s.sm_count = prop.multiProcessorCount;
        s.cc_major = prop.major;
        s.cc_minor = prop.minor;
        int khz = 0;
        if (cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess || khz <= 0) khz = 2000000;
        s.clock_khz = khz;
        if (cudaMalloc(&s.err, sizeof(int)) != cudaSuccess) return GQA_ERR_CUDA;
        if (cudaMemset(s.err, 0, sizeof(int)) != cudaSuccess) return GQA_ERR_CUDA;
        s.init = true;
    }
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return GQA_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = &s;
    return GQA_OK;
}

// 2-D byte view [rows, cols] (E4M3 K/V) with a (cols x box_rows) box and the
// 128-byte swizzle; cols = 128 bytes = one swizzle row.
int make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(cols), box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_CUDA;
}

// 2-D bf16 view [rows, cols] with a (64 x box_rows) box and the 128-byte swizzle.
int make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                 float scale) {
    if (B < 0 || Tq < 0 || Hq <= 0 || Hkv <= 0 || Tkv < 1) return GQA_ERR_SHAPE;
    if (!(scale > 0.f) || !std::isfinite(scale)) return GQA_ERR_SHAPE;
    if (Hq % Hkv != 0) return GQA_ERR_SHAPE;
    if (d != 64 && d != 128 && d != 256 && d != 512) return GQA_ERR_UNSUPPORTED;
    const long long qrows = static_cast<long long>(B) * Hq * Tq;
    const long long kvrows = static_cast<long long>(B) * Hkv * Tkv;
    if (qrows + BM >= (1ll << 31) || kvrows + 256 >= (1ll << 31)) return GQA_ERR_SHAPE;
    if (B == 0 || Tq == 0) return GQA_OK;
    if (!q || !k || !v) return GQA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return GQA_ERR_ALIGN;
    return GQA_OK;
}

void fill_params(Params& p, int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale, int causal,
                 const int32_t* kv_lens, const float* sink, void* out, float* lse, int BN, long long timeout) {
    std::memset(&p, 0, sizeof p);
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Tq = Tq;
    p.Tkv = Tkv;
    p.d = d;
    p.G = Hq / Hkv;
    p.R = p.G * Tq;
    p.QT = (p.R + BM - 1) / BM;
    p.U = B * Hkv;
    p.RBQ = 1;
    p.QW = p.QT;
    p.W = static_cast<long long>(p.U) * p.QW;
    p.causal = causal ? 1 : 0;
    p.BN = BN;
    p.scale_log2 = scale * LOG2E;
    p.kv_lens = kv_lens;
    p.sink = sink;
    p.out = reinterpret_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.timeout_cycles = timeout;
    p.kv_fp8 = 0;
    p.v_scale = 1.f;
}

// Kernel configurations (shared-memory and TMEM budgets are checked in the Cfg
// structs).  Head dims 64 and 128 use the two-lane kernel: split-key lanes when
// a unit's packed rows fit one 128-row q-tile (decode, short-q), dual-Q lanes
// (two q-tiles per row-block sharing every K/V tile) otherwise.  Head dim 256
// keeps one O accumulator (256 TMEM columns) and uses the single-lane kernel.
using C2_64_SK = Fwd2Cfg<64, 4, 4, 1>;
using C2_64_DQ = Fwd2Cfg<64, 4, 4, 2>;
using C2_128_SK = Fwd2Cfg<128, 3, 3, 1>;
using C2_128_DQ = Fwd2Cfg<128, 3, 2, 2>;
// the same four over a paged K/V cache (a separate instantiation keeps the
// page-table producer out of the contiguous kernels)
using C2_64_SK_P = Fwd2Cfg<64, 4, 4, 1, true>;
using C2_64_DQ_P = Fwd2Cfg<64, 4, 4, 2, true>;
using C2_128_SK_P = Fwd2Cfg<128, 3, 3, 1, true>;
using C2_128_DQ_P = Fwd2Cfg<128, 3, 2, 2, true>;
// Few packed rows (decode) at head dim 128: the swap-AB kernel, reading 8 or 16
// rows of its transposed tiles
using CDec8 = DecCfg<8>;
using CDec16 = DecCfg<16>;
using CDec8_P = DecCfg<8, true>;
using CDec16_P = DecCfg<16, true>;
// the same over an E4M3 K/V cache (converted to f16 in shared memory)
using CDec8_F8 = DecCfg<8, false, true>;
using CDec16_F8 = DecCfg<16, false, true>;
bool uses_decode_kernel(const Params& p) { return p.d == 128 && p.mode == 0 && p.R <= DEC_NQ; }
// Head dims 256 and 512: the wide kernel (128-key tiles streamed in 64-column
// chunks past a resident Q tile, in-kernel merge of split row-blocks).  At 512 a
// 128 x 512 fp32 O fills a whole TMEM, so O's columns are split over a pair of
// CTAs (DSPLIT = 2) that each compute the full S.
using CW256 = WideCfg<256, 1>;
using CW512 = WideCfg<512, 2>;

int dsplit_for(int d) { return d == 512 ? CW512::DSPLIT : 1; }

// Tile geometry of the kernel that will serve these sizes.
// Extra weight (in key tiles) of a row-block start when the swap-AB decode
// kernel cuts the work into spans: a segment's epilogue, switch and merge share
// against a tile's streaming time.  Measured on the batched decode (B = 16, ragged
// lengths): 7 tiles for bf16 K/V (1.25 us per tile; 85 -> 78 us against equal
// spans), 2 for E4M3 K/V (its tiles take 1.75 us; 79 -> 69 us).
int seg_weight(bool fp8) {
    if (const char* e = std::getenv("GQA_SEG_WEIGHT")) {
        const int v = std::atoi(e);
        if (v >= 0 && v <= 64) return v;
    }
    return fp8 ? 2 : 7;
}

void choose_geometry(Params& p) {
    p.BN = 128;
    p.RBQ = (p.d <= 128 && p.R > BM) ? 2 : 1;
    p.QW = (p.QT + p.RBQ - 1) / p.RBQ;
    p.W = static_cast<long long>(p.U) * p.QW;
    p.seg_w = (p.d == 128 && p.R <= DEC_NQ && p.B <= kMaxWeightedB) ? seg_weight(p.kv_fp8 != 0) : 0;
}

// Kernel families: the wide kernel (head dims 256, 512), the two-lane kernel
// (64, 128) and the swap-AB decode kernel (128, at most 16 packed rows).
enum KernelKind { kWide = 0, kTwoLane = 1, kDecode = 2 };

template <class C, int KIND>
int launch_fwd(const Params& p0, const void* q, const void* k, const void* v, int grid, cudaStream_t stream,
               cudaEvent_t ev_before, cudaEvent_t ev_after) {
    static bool attr_done[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
    if (!attr_done[dev]) {
        cudaError_t e;
        if constexpr (KIND == kTwoLane)
            e = cudaFuncSetAttribute(gqa_fwd2_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        else if constexpr (KIND == kDecode)
            e = cudaFuncSetAttribute(gqa_dec_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        else
            e = cudaFuncSetAttribute(gqa_wide_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return GQA_ERR_CUDA;
        attr_done[dev] = true;
    }
    CUtensorMap tq, tk, tv;
    Params p = p0;
    // a box never taller than the tensor; rows a short box leaves unwritten are
    // padding rows (query rows past the group, or key rows past kv_len, which the
    // kernel zeroes in V and masks in S)
    const uint64_t qrows = static_cast<uint64_t>(p.B) * p.Hq * p.Tq;
    // paged K/V: the caches viewed as [num_pages*Hkv*page_size, d], one box per page piece
    const bool paged = p.page_size > 0;
    const uint64_t kvrows = paged ? static_cast<uint64_t>(p.num_pages) * p.Hkv * p.page_size
                                  : static_cast<uint64_t>(p.B) * p.Hkv * p.Tkv;
    const uint64_t kvcols = static_cast<uint64_t>(C::D);
    // few packed rows (decode): spread them over the four TMEM lane quadrants so
    // that every SM sub-partition takes a share of the softmax
    p.spread = (KIND == kTwoLane && p.QT == 1 && p.R <= 96) ? 1 : 0;
    p.rq = (p.R + 3) / 4;
    if constexpr (KIND == kDecode)  // the 16-row Q tile of the transposed MMAs
        p.q_box_rows = qrows < static_cast<uint64_t>(DEC_NQ) ? static_cast<int>(qrows) : DEC_NQ;
    else
        p.q_box_rows = p.spread ? p.rq : (qrows < static_cast<uint64_t>(BM) ? static_cast<int>(qrows) : BM);
    if (paged)
        p.kv_box_rows = p.page_size < C::BN ? p.page_size : C::BN;
    else
        p.kv_box_rows = kvrows < static_cast<uint64_t>(C::BN) ? static_cast<int>(kvrows) : C::BN;
    int rc = make_tmap(&tq, q, qrows, C::D, p.q_box_rows);
    if (rc) return rc;
    if constexpr (KIND == kDecode && C::FP8) {
        rc = make_tmap_u8(&tk, k, kvrows, kvcols, p.kv_box_rows);
        if (rc) return rc;
        rc = make_tmap_u8(&tv, v, kvrows, kvcols, p.kv_box_rows);
        if (rc) return rc;
    } else {
        rc = make_tmap(&tk, k, kvrows, kvcols, p.kv_box_rows);
        if (rc) return rc;
        rc = make_tmap(&tv, v, kvrows, kvcols, p.kv_box_rows);
        if (rc) return rc;
    }
    if (ev_before && cudaEventRecord(ev_before, stream) != cudaSuccess) return GQA_ERR_CUDA;
    if constexpr (KIND == kTwoLane)
        gqa_fwd2_kernel<C><<<grid, NUM_THREADS2, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    else if constexpr (KIND == kDecode)
        gqa_dec_kernel<C><<<grid, C::NTHREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    else {
        // the stream-K merge waits for pieces written by other CTAs of the grid:
        // every CTA must be resident at once, which a cooperative launch guarantees
        // (or refuses); the uniform splits of mode 1 never wait on another CTA
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(NUM_THREADS_W);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = (p.mode == 0) ? 1 : 0;
        if (cudaLaunchKernelEx(&cfg, gqa_wide_kernel<C>, tq, tk, tv, p) != cudaSuccess) return GQA_ERR_CUDA;
    }
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
    if (ev_after && cudaEventRecord(ev_after, stream) != cudaSuccess) return GQA_ERR_CUDA;
    return GQA_OK;
}

int dispatch_fwd(const Params& p, const void* q, const void* k, const void* v, int grid, cudaStream_t stream,
                 cudaEvent_t e0 = nullptr, cudaEvent_t e1 = nullptr) {
    switch (p.d) {
        case 64:
            if (p.page_size > 0)
                return p.RBQ == 1 ? launch_fwd<C2_64_SK_P, kTwoLane>(p, q, k, v, grid, stream, e0, e1)
                                  : launch_fwd<C2_64_DQ_P, kTwoLane>(p, q, k, v, grid, stream, e0, e1);
            return p.RBQ == 1 ? launch_fwd<C2_64_SK, kTwoLane>(p, q, k, v, grid, stream, e0, e1)
                              : launch_fwd<C2_64_DQ, kTwoLane>(p, q, k, v, grid, stream, e0, e1);
        case 128:
            if (uses_decode_kernel(p)) {
                if (p.kv_fp8)
                    return p.R <= 8 ? launch_fwd<CDec8_F8, kDecode>(p, q, k, v, grid, stream, e0, e1)
                                    : launch_fwd<CDec16_F8, kDecode>(p, q, k, v, grid, stream, e0, e1);
                if (p.page_size > 0)
                    return p.R <= 8 ? launch_fwd<CDec8_P, kDecode>(p, q, k, v, grid, stream, e0, e1)
                                    : launch_fwd<CDec16_P, kDecode>(p, q, k, v, grid, stream, e0, e1);
                return p.R <= 8 ? launch_fwd<CDec8, kDecode>(p, q, k, v, grid, stream, e0, e1)
                                : launch_fwd<CDec16, kDecode>(p, q, k, v, grid, stream, e0, e1);
            }
            if (p.page_size > 0)
                return p.RBQ == 1 ? launch_fwd<C2_128_SK_P, kTwoLane>(p, q, k, v, grid, stream, e0, e1)
                                  : launch_fwd<C2_128_DQ_P, kTwoLane>(p, q, k, v, grid, stream, e0, e1);
            return p.RBQ == 1 ? launch_fwd<C2_128_SK, kTwoLane>(p, q, k, v, grid, stream, e0, e1)
                              : launch_fwd<C2_128_DQ, kTwoLane>(p, q, k, v, grid, stream, e0, e1);
        case 256: return launch_fwd<CW256, kWide>(p, q, k, v, grid, stream, e0, e1);
        case 512: return launch_fwd<CW512, kWide>(p, q, k, v, grid, stream, e0, e1);
        default: return GQA_ERR_UNSUPPORTED;
    }
}

// About one second of SM clock for every wait inside the kernels; tests shorten
// it with GQA_WAIT_TIMEOUT_US (microseconds) or GQA_WAIT_TIMEOUT_MS.
long long wait_limit_cycles(long long clock_khz) {
    if (const char* e = std::getenv("GQA_WAIT_TIMEOUT_US")) {
        const long long us = std::atoll(e);
        if (us > 0) return clock_khz * us / 1000;
    }
    long long ms = 1000;
    if (const char* e = std::getenv("GQA_WAIT_TIMEOUT_MS")) {
        const long long v = std::atoll(e);
        if (v > 0) ms = v;
    }
    return clock_khz * ms;
}
long long timeout_cycles(const DeviceState& s) { return wait_limit_cycles(s.clock_khz); }

int ensure_counters(DeviceState& s, long long n) {
    if (s.counters_len >= n) return GQA_OK;
    if (s.counters) {
        if (cudaDeviceSynchronize() != cudaSuccess) return GQA_ERR_CUDA;
        cudaFree(s.counters);
        s.counters = nullptr;
        s.counters_len = 0;
    }
    long long len = n < 4096 ? 4096 : n;
    if (cudaMalloc(&s.counters, sizeof(int) * static_cast<size_t>(len)) != cudaSuccess) return GQA_ERR_CUDA;
    if (cudaMemset(s.counters, 0, sizeof(int) * static_cast<size_t>(len)) != cudaSuccess) return GQA_ERR_CUDA;
    s.counters_len = len;
    return GQA_OK;
}

int ensure_scratch(DeviceState& s, size_t bytes) {
    if (s.scratch_bytes >= bytes) return GQA_OK;
    if (s.scratch) {
        // the old buffer may still be read by work queued on any stream
        if (cudaDeviceSynchronize() != cudaSuccess) return GQA_ERR_CUDA;
        cudaFree(s.scratch);
        s.scratch = nullptr;
        s.scratch_bytes = 0;
    }
    if (cudaMalloc(&s.scratch, bytes) != cudaSuccess) return GQA_ERR_CUDA;
    s.scratch_bytes = bytes;
    return GQA_OK;
}

// The stream-K forward shared by the contiguous and the paged entry points:
// plan, scratch, launch (and the combine launch for head dims 256 / 512).
int run_streamk(Params& p, const void* q, const void* k, const void* v, DeviceState& sr, gqa_stream_t stream) {
    DeviceState* s = &sr;
    const int d = p.d, Tkv = p.Tkv;
    const bool has_lens = p.kv_lens != nullptr;
    int rc = GQA_OK;
    choose_geometry(p);
    // grid: one CTA per SM (NC groups of DSPLIT CTAs); with host-known lengths never
    // more groups than tiles
    const int ds = dsplit_for(d);
    int NC = (s->sm_count < kMaxCtas ? s->sm_count : kMaxCtas) / ds;
    if (!has_lens) {
        long long tot = 0;
        for (int qw = 0; qw < p.QW; ++qw) tot += qtile_ntiles(p, qw, Tkv);
        tot *= p.U;
        if (tot < NC) NC = static_cast<int>(tot);
    }
    if (NC < 1) NC = 1;
    const size_t slot_rows = static_cast<size_t>(2 * NC) * ds * BM * p.RBQ;
    const size_t slot_o = slot_rows * (d / ds) * sizeof(float);
    const size_t slot_l = (slot_rows * sizeof(float) + 255) & ~static_cast<size_t>(255);
    // merge counters: one ticket per row-block (head dims <= 128), a published /
    // merged pair per row-block and O part (256, 512)
    const long long nctr = 2 * p.W * ds + 2;
    cudaStream_t st0 = reinterpret_cast<cudaStream_t>(stream);
    if (s->scratch_bytes < slot_o + slot_l || s->counters_len < nctr) {
        // growing the scratch allocates (and synchronises): not while the stream is
        // being captured into a CUDA graph
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(st0, &cs) != cudaSuccess) return GQA_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone) return GQA_ERR_SCRATCH;
    }
    rc = ensure_scratch(*s, slot_o + slot_l);
    if (rc) return rc;
    rc = ensure_counters(*s, nctr);
    if (rc) return rc;
    char* base = static_cast<char*>(s->scratch);
    p.mode = 0;
    p.part_o = reinterpret_cast<float*>(base);
    p.part_lse = reinterpret_cast<float*>(base + slot_o);
    p.counters = s->counters;
    p.err = s->err;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaEvent_t* ev = nullptr;
    if (g_prof.on && g_prof.n < kProfCap) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev == g_prof.dev) ev = g_prof.ev[g_prof.n++];
    }
    rc = dispatch_fwd(p, q, k, v, NC * ds, st, ev ? ev[0] : nullptr, ev ? ev[1] : nullptr);
    if (rc) return rc;
    return GQA_OK;
}

}  // namespace
}  // namespace gqa

using namespace gqa;

extern "C" int gqa_attention_fwd(const void* q, const void* k, const void* v, const int32_t* kv_lens,
                                 const float* sink, void* out, float* lse, int B, int Hq, int Hkv, int Tq,
                                 int Tkv, int d, float scale, int causal, gqa_stream_t stream) {
    int rc = check_common(q, k, v, B, Hq, Hkv, Tq, Tkv, d, scale);
    if (rc) return rc;
    if (B == 0 || Tq == 0) return GQA_OK;
    if (!out) return GQA_ERR_NULL;
    if (!aligned16(out) || (lse && !aligned16(lse))) return GQA_ERR_ALIGN;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState* s = nullptr;
    rc = get_state(&s);
    if (rc) return rc;
    if (s->cc_major != 10) return GQA_ERR_UNSUPPORTED;
    Params p;
    fill_params(p, B, Hq, Hkv, Tq, Tkv, d, scale, causal, kv_lens, sink, out, lse, 0, timeout_cycles(*s));
    return run_streamk(p, q, k, v, *s, stream);
}

extern "C" int gqa_attention_fwd_fp8kv(const void* q, const void* k8, const void* v8, float k_scale, float v_scale,
                                       const int32_t* kv_lens, const float* sink, void* out, float* lse, int B, int Hq,
                                       int Hkv, int Tq, int Tkv, int d, float scale, int causal, gqa_stream_t stream) {
    int rc = check_common(q, k8, v8, B, Hq, Hkv, Tq, Tkv, d, scale);
    if (rc) return rc;
    if (!(k_scale > 0.f) || !std::isfinite(k_scale) || !(v_scale > 0.f) || !std::isfinite(v_scale)) return GQA_ERR_SHAPE;
    // the swap-AB decode kernel's shapes: head dim 128, at most 16 packed rows per KV head
    if (d != 128 || (Hq / Hkv) * static_cast<long long>(Tq) > DEC_NQ) return GQA_ERR_UNSUPPORTED;
    if (!std::isfinite(scale * k_scale)) return GQA_ERR_SHAPE;
    if (B == 0 || Tq == 0) return GQA_OK;
    if (!out) return GQA_ERR_NULL;
    if (!aligned16(out) || (lse && !aligned16(lse))) return GQA_ERR_ALIGN;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState* s = nullptr;
    rc = get_state(&s);
    if (rc) return rc;
    if (s->cc_major != 10) return GQA_ERR_UNSUPPORTED;
    Params p;
    fill_params(p, B, Hq, Hkv, Tq, Tkv, d, scale * k_scale, causal, kv_lens, sink, out, lse, 0, timeout_cycles(*s));
    p.kv_fp8 = 1;
    p.v_scale = v_scale;
    return run_streamk(p, q, k8, v8, *s, stream);
}

extern "C" int gqa_attention_fwd_paged(const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* page_table, const int32_t* kv_lens, const float* sink, void* out,
                                       float* lse, int B, int Hq, int Hkv, int Tq, int num_pages, int page_size,
                                       int max_pages, int d, float scale, int causal, gqa_stream_t stream) {
    if (page_size < 8 || page_size > 1024 || (page_size & (page_size - 1)) != 0) return GQA_ERR_SHAPE;
    if (num_pages < 1 || max_pages < 1) return GQA_ERR_SHAPE;
    if (static_cast<long long>(max_pages) * page_size >= (1ll << 30)) return GQA_ERR_SHAPE;
    if (static_cast<long long>(num_pages) * (Hkv > 0 ? Hkv : 1) * page_size + 256 >= (1ll << 31)) return GQA_ERR_SHAPE;
    const int Tkv = max_pages * page_size;  // a sequence's capacity
    int rc = check_common(q, k_cache, v_cache, B, Hq, Hkv, Tq, Tkv, d, scale);
    if (rc) return rc;
    if (d != 64 && d != 128) return GQA_ERR_UNSUPPORTED;
    if (B == 0 || Tq == 0) return GQA_OK;
    if (!out || !page_table || !kv_lens) return GQA_ERR_NULL;
    if (!aligned16(out) || (lse && !aligned16(lse))) return GQA_ERR_ALIGN;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState* s = nullptr;
    rc = get_state(&s);
    if (rc) return rc;
    if (s->cc_major != 10) return GQA_ERR_UNSUPPORTED;
    Params p;
    fill_params(p, B, Hq, Hkv, Tq, Tkv, d, scale, causal, kv_lens, sink, out, lse, 0, timeout_cycles(*s));
    p.page_table = page_table;
    p.page_size = page_size;
    p.max_pages = max_pages;
    p.num_pages = num_pages;
    return run_streamk(p, q, k_cache, v_cache, *s, stream);
}

extern "C" int gqa_attention_fwd_partial(const void* q, const void* k, const void* v, const int32_t* kv_lens,
                                         int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale, int causal,
                                         int num_splits, float* o_part, float* lse_part, gqa_stream_t stream) {
    int rc = check_common(q, k, v, B, Hq, Hkv, Tq, Tkv, d, scale);
    if (rc) return rc;
    if (num_splits < 1 || num_splits > GQA_MAX_SPLITS) return GQA_ERR_SPLITS;
    if (B == 0 || Tq == 0) return GQA_OK;
    if (!o_part || !lse_part) return GQA_ERR_NULL;
    if (!aligned16(o_part) || !aligned16(lse_part)) return GQA_ERR_ALIGN;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState* s = nullptr;
    rc = get_state(&s);
    if (rc) return rc;
    if (s->cc_major != 10) return GQA_ERR_UNSUPPORTED;
    Params p;
    fill_params(p, B, Hq, Hkv, Tq, Tkv, d, scale, causal, kv_lens, nullptr, nullptr, nullptr, 0,
                timeout_cycles(*s));
    choose_geometry(p);
    const long long grid = p.W * num_splits * dsplit_for(d);
    if (grid >= (1ll << 31)) return GQA_ERR_SHAPE;
    p.mode = 1;
    p.num_splits = num_splits;
    p.part_o = o_part;
    p.part_lse = lse_part;
    p.err = s->err;
    return dispatch_fwd(p, q, k, v, static_cast<int>(grid), reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int gqa_splitkv_combine(const float* o_part, const float* lse_part, int num_splits, const float* sink,
                                   void* out, float* lse, int B, int Hq, int Tq, int d, gqa_stream_t stream) {
    if (B < 0 || Hq <= 0 || Tq < 0 || d <= 0 || d % 4 != 0) return GQA_ERR_SHAPE;
    if (num_splits < 1 || num_splits > GQA_MAX_SPLITS) return GQA_ERR_SPLITS;
    if (B == 0 || Tq == 0) return GQA_OK;
    if (!o_part || !lse_part || !out) return GQA_ERR_NULL;
    if (!aligned16(o_part) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse_part) & 3u)) return GQA_ERR_ALIGN;
    const long long rows = static_cast<long long>(B) * Hq * Tq;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState* s = nullptr;
    int rc = get_state(&s);
    if (rc) return rc;
    long long blocks = (rows + 7) / 8;
    const long long cap = static_cast<long long>(s->sm_count) * 16;
    if (blocks > cap) blocks = cap;
    const size_t smem = static_cast<size_t>(8) * num_splits * sizeof(float);
    gqa_combine_uniform_kernel<<<static_cast<int>(blocks), 256, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
        o_part, lse_part, num_splits, sink, reinterpret_cast<__nv_bfloat16*>(out), lse, rows, Hq, Tq, d);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

extern "C" int gqa_shard_lengths(const int32_t* kv_lens, int B, int key_offset, int shard_capacity,
                                 int32_t* shard_lens, gqa_stream_t stream) {
    if (B < 0 || key_offset < 0 || shard_capacity < 0) return GQA_ERR_SHAPE;
    if (B == 0) return GQA_OK;
    if (!kv_lens || !shard_lens) return GQA_ERR_NULL;
    const int blocks = (B + 255) / 256 < 1024 ? (B + 255) / 256 : 1024;
    gqa_shard_lengths_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(kv_lens, B, key_offset,
                                                                                      shard_capacity, shard_lens);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

extern "C" int gqa_combine_shards(const void* o_shards, long long o_shard_stride, const float* lse_shards,
                                  long long lse_shard_stride, int num_shards, const float* sink, void* out, float* lse,
                                  int B, int Hq, int Tq, int d, gqa_stream_t stream) {
    if (B < 0 || Hq <= 0 || Tq < 0 || d <= 0 || d % 4 != 0) return GQA_ERR_SHAPE;
    if (num_shards < 1 || num_shards > GQA_MAX_SPLITS) return GQA_ERR_SPLITS;
    if (B == 0 || Tq == 0) return GQA_OK;
    if (!o_shards || !lse_shards || !out) return GQA_ERR_NULL;
    const long long rows = static_cast<long long>(B) * Hq * Tq;
    if (num_shards > 1 && (o_shard_stride < rows * d || lse_shard_stride < rows)) return GQA_ERR_SHAPE;
    // four bf16 (8 bytes) per load: the shards' starts stay 8-byte aligned
    if (!aligned16(o_shards) || (o_shard_stride & 3) != 0 || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(lse_shards) & 3u))
        return GQA_ERR_ALIGN;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState* s = nullptr;
    int rc = get_state(&s);
    if (rc) return rc;
    long long blocks = (rows + 7) / 8;
    const long long cap = static_cast<long long>(s->sm_count) * 16;
    if (blocks > cap) blocks = cap;
    const size_t smem = static_cast<size_t>(8) * num_shards * sizeof(float);
    gqa_combine_shards_kernel<<<static_cast<int>(blocks), 256, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const __nv_bfloat16*>(o_shards), o_shard_stride, lse_shards, lse_shard_stride, num_shards, sink,
        reinterpret_cast<__nv_bfloat16*>(out), lse, rows, Hq, Tq, d);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

extern "C" int gqa_profile_begin(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
    if (g_prof.created && g_prof.dev != dev) {
        for (auto& e : g_prof.ev)
            for (auto& x : e) cudaEventDestroy(x);
        g_prof.created = false;
    }
    if (!g_prof.created) {
        for (auto& e : g_prof.ev)
            for (auto& x : e)
                if (cudaEventCreate(&x) != cudaSuccess) return GQA_ERR_CUDA;
        g_prof.created = true;
    }
    g_prof.dev = dev;
    g_prof.n = 0;
    g_prof.on = true;
    return GQA_OK;
}

extern "C" int gqa_profile_take(float* kernel_ms, int max_calls, int* n_calls) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!n_calls) return GQA_ERR_NULL;
    g_prof.on = false;
    const int n = g_prof.n < max_calls ? g_prof.n : max_calls;
    for (int i = 0; i < n; ++i) {
        if (cudaEventSynchronize(g_prof.ev[i][1]) != cudaSuccess) return GQA_ERR_CUDA;
        float a = 0.f;
        if (cudaEventElapsedTime(&a, g_prof.ev[i][0], g_prof.ev[i][1]) != cudaSuccess) return GQA_ERR_CUDA;
        if (kernel_ms) kernel_ms[i] = a;
    }
    *n_calls = n;
    g_prof.n = 0;
    return GQA_OK;
}

extern "C" const char* gqa_status_string(int status) {
    switch (status) {
        case GQA_OK: return "ok";
        case GQA_ERR_NULL: return "a required pointer is NULL";
        case GQA_ERR_SHAPE: return "invalid shape";
        case GQA_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case GQA_ERR_SPLITS: return "num_splits out of range";
        case GQA_ERR_CUDA: return "a CUDA call failed";
        case GQA_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
        case GQA_ERR_UNSUPPORTED: return "unsupported head dim or GPU";
        case GQA_ERR_KVLEN: return "a kv_lens value was outside [0, Tkv] and was clamped";
        case GQA_ERR_PAGE: return "a page id was outside [0, num_pages); page 0 was read instead";
        case GQA_ERR_SMEM_ALIGN: return "a kernel's dynamic shared memory was not 1024-byte aligned (internal error)";
        case GQA_ERR_SCRATCH:
            return "the problem needs more scratch than is in place (the allocation-free array, or a call being "
                   "captured into a CUDA graph before an uncaptured call of that size)";
        default: return "unknown status";
    }
}

extern "C" int gqa_version(void) { return 100; }

// ---------------------------------------------------------------------------
// Allocation-free variant of gqa_attention_fwd.
//
// gqa_attention_fwd grows a per-device scratch buffer with cudaMalloc the first
// time it meets a problem that needs more room.  Some callers cannot allow that:
// an engine that hands all device memory to its own pools at start-up and must
// not see the driver allocate behind its back, a caller running inside a section
// where an allocation (which may synchronise the device) is forbidden, or a host
// integration that has no allocator at all.  For them this entry point keeps the
// split-partial scratch in one fixed array compiled into this library, so every
// GPU that loads the library holds it until the process exits.
namespace gqa {
namespace {

constexpr size_t kNaCounterInts = 65536;                         // merge counters
constexpr size_t kNaErrOffset = kNaCounterInts * sizeof(int);    // device error word
constexpr size_t kNaLseOffset = kNaErrOffset + 256;
constexpr size_t kNaLseFloats = static_cast<size_t>(2) * kMaxCtas * 2 * BM;  // 2 slots x 256 rows per CTA
constexpr size_t kNaPartOffset = kNaLseOffset + kNaLseFloats * sizeof(float);
constexpr size_t kNaPartBytes = static_cast<size_t>(20) << 20;  // fp32 partial O: 20 MiB
constexpr size_t kNaBytes = kNaPartOffset + kNaPartBytes;       // about 21.3 MiB in all

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaBytes];

struct NoAllocDevice {
    bool ready = false;
    unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch on this device
    int sm_count = 0;
    int cc_major = 0;
    long long clock_khz = 0;
};
NoAllocDevice g_na_dev[kMaxDevices];

// Once per device, with that device current: the array's device address (the
// host-side name g_noalloc_scratch is only a stand-in, not an address a kernel
// may use), the SM count and clock, and the tensor-map encoder.
int noalloc_setup(NoAllocDevice** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
    NoAllocDevice& s = g_na_dev[dev];
    if (!s.ready) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return GQA_ERR_CUDA;
        int sms = 0, major = 0, khz = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return GQA_ERR_CUDA;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return GQA_ERR_CUDA;
        if (cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess || khz <= 0) khz = 2000000;
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return GQA_ERR_CUDA;
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        s.scratch = static_cast<unsigned char*>(ptr);
        s.sm_count = sms;
        s.cc_major = major;
        s.clock_khz = khz;
        s.ready = true;
    }
    *out = &s;
    return GQA_OK;
}

}  // namespace
}  // namespace gqa

extern "C" int gqa_attention_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* kv_lens,
                                         const float* sink, void* out, float* lse, int B, int Hq, int Hkv, int Tq,
                                         int Tkv, int d, float scale, int causal, gqa_stream_t stream) {
    int rc = check_common(q, k, v, B, Hq, Hkv, Tq, Tkv, d, scale);
    if (rc) return rc;
    if (B == 0 || Tq == 0) return GQA_OK;
    if (!out) return GQA_ERR_NULL;
    if (!aligned16(out) || (lse && !aligned16(lse))) return GQA_ERR_ALIGN;
    std::lock_guard<std::mutex> lk(g_mu);
    NoAllocDevice* s = nullptr;
    rc = noalloc_setup(&s);
    if (rc) return rc;
    if (s->cc_major != 10) return GQA_ERR_UNSUPPORTED;
    Params p;
    fill_params(p, B, Hq, Hkv, Tq, Tkv, d, scale, causal, kv_lens, sink, out, lse, 0, wait_limit_cycles(s->clock_khz));
    choose_geometry(p);
    const int ds = dsplit_for(d);
    // merge counters: a ticket per row-block (head dims <= 128), a published /
    // merged pair per row-block and O part (256, 512)
    const long long nctr = (d >= 256) ? 2 * p.W * ds : p.W;
    if (nctr > static_cast<long long>(kNaCounterInts)) return GQA_ERR_SCRATCH;
    // as many CTA groups (one CTA per SM) as the fixed partial area can give two slots each
    const size_t rows_per_slot = static_cast<size_t>(BM) * p.RBQ;
    const size_t per_group = 2 * rows_per_slot * static_cast<size_t>(d) * sizeof(float);
    long long NC = (s->sm_count < kMaxCtas ? s->sm_count : kMaxCtas) / ds;
    if (static_cast<long long>(kNaPartBytes / per_group) < NC) NC = static_cast<long long>(kNaPartBytes / per_group);
    if (!kv_lens) {
        long long tot = 0;
        for (int qw = 0; qw < p.QW; ++qw) tot += qtile_ntiles(p, qw, Tkv);
        tot *= p.U;
        if (tot < NC) NC = tot;
    }
    if (NC < 1) return GQA_ERR_SCRATCH;
    unsigned char* base = s->scratch;
    p.mode = 0;
    p.part_o = reinterpret_cast<float*>(base + kNaPartOffset);
    p.part_lse = reinterpret_cast<float*>(base + kNaLseOffset);
    p.counters = reinterpret_cast<int*>(base);
    p.err = reinterpret_cast<int*>(base + kNaErrOffset);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the array keeps the last call's contents: the merge counters and the error
    // word must start at zero
    if (cudaMemsetAsync(base, 0, static_cast<size_t>(nctr) * sizeof(int), st) != cudaSuccess) return GQA_ERR_CUDA;
    if (cudaMemsetAsync(base + kNaErrOffset, 0, 32, st) != cudaSuccess) return GQA_ERR_CUDA;
    rc = dispatch_fwd(p, q, k, v, static_cast<int>(NC * ds), st);
    if (rc) return rc;
    return GQA_OK;
}

// Reads (and clears) the device error words of the current device: the
// allocating entry points' word (only if they have run here: reading it never
// allocates) and the fixed array's word of the allocation-free entry point
// (only if it has run here).  The first non-zero word is returned.
extern "C" int gqa_get_device_error(gqa_stream_t stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return GQA_ERR_CUDA;
    int first = 0;
    DeviceState& s = g_dev[dev];
    if (s.init) {
        int v = 0;
        if (cudaMemcpy(&v, s.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GQA_ERR_CUDA;
        if (v != 0) {
            if (cudaMemset(s.err, 0, sizeof(int)) != cudaSuccess) return GQA_ERR_CUDA;
            // an aborted launch may leave merge tickets behind
            if (s.counters && cudaMemset(s.counters, 0, sizeof(int) * static_cast<size_t>(s.counters_len)) != cudaSuccess)
                return GQA_ERR_CUDA;
            first = v;
        }
    }
    const NoAllocDevice& na = g_na_dev[dev];
    if (na.ready) {
        int v = 0;
        if (cudaMemcpy(&v, na.scratch + kNaErrOffset, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
            return GQA_ERR_CUDA;
        if (v != 0) {
            // the error word, the combine-job counters and the merge tickets (each
            // call clears the tickets it uses, but an aborted launch may leave
            // others behind)
            if (cudaMemset(na.scratch + kNaErrOffset, 0, 32) != cudaSuccess) return GQA_ERR_CUDA;
            if (cudaMemset(na.scratch, 0, kNaCounterInts * sizeof(int)) != cudaSuccess) return GQA_ERR_CUDA;
            if (first == 0) first = v;
        }
    }
    return first;
}

