// C-ABI entry points of the W4A16 library: argument validation, launch
// planning, TMA descriptors, dispatch.  Declared in include/w4a16.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gemm_simple.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "gemv_mma.cuh"
#include "gemv_q8.cuh"
#include "gemv_t_mma.cuh"
#include "permute.cuh"
#include "quantize.cuh"
#include "w4a16.h"

namespace {

using namespace w4;

thread_local cudaError_t g_last_cuda_error = cudaSuccess;
std::atomic<int> g_debug_checks{0};

// ----------------------------------------------------------------- device info
struct DeviceInfo {
    int sms = 0;
    int max_smem_optin = 0;
};

DeviceInfo device_info(int dev) {
    static std::mutex mu;
    static DeviceInfo cache[64];
    static bool have[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && have[dev]) return cache[dev];
    DeviceInfo d;
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (d.sms <= 0) {  // no usable device: keep the planners well defined
        cudaGetLastError();
        d.sms = 1;
        d.max_smem_optin = 0;
        return d;
    }
    if (dev >= 0 && dev < 64) {
        cache[dev] = d;
        have[dev] = true;
    }
    return d;
}

int current_device() {
    int dev = 0;
    cudaGetDevice(&dev);
    return dev;
}

// Raise a kernel's dynamic shared-memory limit once per (device, kernel).
cudaError_t ensure_smem(const void* fn, size_t bytes) {
    static std::mutex mu;
    struct Entry {
        int dev;
        const void* fn;
        size_t bytes;
    };
    static Entry table[512];
    static int count = 0;
    const int dev = current_device();
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < count; ++i)
        if (table[i].dev == dev && table[i].fn == fn && table[i].bytes >= bytes) return cudaSuccess;
    cudaError_t e =
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        cudaGetLastError();
        return e;
    }
    if (count < 512) table[count++] = Entry{dev, fn, bytes};
    return cudaSuccess;
}

// Launch `fn` as a programmatic dependent of the work before it on `st`:
// it may start once that work has let it (griddepcontrol.launch_dependents)
// and must wait (griddepcontrol.wait) before reading that work's results.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*fn)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, fn, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major tensor [rows, cols] of `esize`-byte elements, box [box_rows,
// box_cols], swizzle span 0 (none), 64 or 128 bytes.  Out-of-range elements
// read as 0.
bool make_map_2d(CUtensorMap* map, const void* ptr, CUtensorMapDataType dt, int esize,
                 uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                 int swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols * static_cast<uint64_t>(esize)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void*>(ptr), gdim, gstride, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                    : swizzle == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                    : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// n `esize`-byte elements as a one-row 2-D tensor (the row stride is never
// stepped; it is only rounded up to the 16 bytes the encoder requires), box
// of `box` elements.
bool make_map_row(CUtensorMap* map, const void* ptr, CUtensorMapDataType dt, int esize, uint64_t n, uint32_t box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[2] = {n, 1};
    cuuint64_t gstride[1] = {(n * esize + 15) / 16 * 16};
    cuuint32_t bx[2] = {box, 1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void*>(ptr), gdim, gstride, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------ validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Meta {
    int g;       // group length along K (K for ROWWISE / GLOBAL)
    int G;       // groups per row
    int sz_row;  // row stride of the scale / zero arrays
    int fmt;     // format flags of the mode (kFmtZeroFloat, kFmtMetaBf16)
};

// The mode argument: a base mode or-ed with format flags.
constexpr int kModeBaseMask = 0x0F;

w4_status check_mode(int K, int mode, int group_size, Meta* meta) {
    const int fmt = mode & ~kModeBaseMask;
    if (fmt & ~(W4_ZERO_FLOAT | W4_META_BF16)) return W4_ERR_INVALID_ARG;
    static_assert(W4_ZERO_FLOAT == kFmtZeroFloat && W4_META_BF16 == kFmtMetaBf16, "format flags");
    switch (mode & kModeBaseMask) {
        case W4_MODE_GLOBAL: *meta = Meta{K, 1, 0, fmt}; return W4_OK;
        case W4_MODE_ROWWISE: *meta = Meta{K, 1, 1, fmt}; return W4_OK;
        case W4_MODE_GROUPWISE:
            if (group_size < 8 || group_size % 8 != 0 || K % group_size != 0) return W4_ERR_INVALID_ARG;
            *meta = Meta{group_size, K / group_size, K / group_size, fmt};
            return W4_OK;
        default: return W4_ERR_INVALID_ARG;
    }
}

std::atomic<uint64_t> g_launches{0};
// Called right after every kernel launch: counts it and maps a launch
// failure to W4_ERR_CUDA (the CUDA error is kept for w4_last_cuda_error).
w4_status launch_status() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return W4_OK;
    g_last_cuda_error = e;
    return W4_ERR_CUDA;
}

// -------------------------------------------------------- GEMV planning
struct TPlan {
    int splits = 1, rows_per_split = 0;
    size_t ws = 0;
};

TPlan plan_t(int M, int N, int K, int sms) {
    TPlan p;
    const int W8 = K / 8;
    const int col_tiles = (W8 + kGemvTWordsPerCta - 1) / kGemvTWordsPerCta;
    int splits = (sms * 6 + col_tiles - 1) / col_tiles;
    splits = std::min(splits, std::max(1, N / (320 * M)));  // partial traffic <= ~5%
    splits = std::max(1, std::min(splits, (N + 31) / 32));
    p.rows_per_split = (N + splits - 1) / splits;
    p.splits = (N + p.rows_per_split - 1) / p.rows_per_split;
    p.ws = p.splits > 1 ? static_cast<size_t>(p.splits) * M * K * sizeof(float) : 0;
    return p;
}

// Tensor-pipe transposed GEMV (gemv_t_mma_kernel): K % 32 == 0 and the
// scale/zero layouts its TMA boxes take (g a multiple of 64 with G % 8 == 0,
// one group per row, or one global pair).  A warp covers KW k of its CTA's
// strip: 128 for M <= 2 when g allows, else 64 (the accumulators of two mma
// column sets then fit).  Row ranges are whole 32-row stages; the grid is a
// whole number of splits per strip, at most one CTA per SM, with the fp32
// partials held under about a tenth of the weights.
struct TMmaPlan {
    bool ok = false;
    int KW = 128, strips = 0, splits = 1, rows_per_split = 0, stages = 0, grid = 0;
    size_t smem = 0, ws = 0;
};

int t_mma_kw(int M, const Meta& meta) {
    return (M <= 2 && (meta.G == 1 || meta.g % 128 == 0)) ? 128 : 64;
}

TMmaPlan plan_t_mma(int M, int N, int K, int KW, int sms, int max_smem) {
    TMmaPlan p;
    p.KW = KW;
    p.strips = (K + tm_strip(KW) - 1) / tm_strip(KW);
    int splits = std::max(1, sms / p.strips);
    splits = std::min(splits, std::max(1, N / (80 * M)));
    splits = std::min(splits, std::max(1, N / (kTMRows * 4)));   // at least 4 stages of rows per split
    auto set_rows = [&](int sp) {
        p.rows_per_split = ((N + sp - 1) / sp + kTMRows - 1) / kTMRows * kTMRows;
        p.splits = (N + p.rows_per_split - 1) / p.rows_per_split;
    };
    set_rows(splits);
    // the split's dY rows live in shared memory: keep them under 32 KB
    while (static_cast<size_t>(p.rows_per_split) * 16 > 32 * 1024) set_rows(++splits);
    p.grid = p.strips * p.splits;
    const int nset = (M + 1) / 2;
    const size_t fixed = gemv_t_mma_smem_bytes(KW, nset, 0, p.rows_per_split);
    const size_t avail = max_smem > 0 ? static_cast<size_t>(max_smem) : 232448;
    p.stages = avail > fixed
                   ? static_cast<int>(std::min<size_t>(8, (avail - fixed) / (tm_stage_bytes(KW) + 16)))
                   : 0;
    p.smem = gemv_t_mma_smem_bytes(KW, nset, p.stages, p.rows_per_split);
    p.ws = p.splits > 1 ? static_cast<size_t>(p.splits) * M * K * sizeof(float) : 0;
    p.ok = p.stages >= 2;
    return p;
}

bool t_mma_eligible(int K, const Meta& meta) {
    if (K % 32 != 0) return false;
    if (meta.sz_row == 0 || meta.G == 1) return true;
    return meta.g % 64 == 0 && meta.G % 8 == 0;
}

// Tensor-pipe forward GEMV (gemv_mma_kernel): K % 32 == 0 and the group
// length a multiple of 32, or one group per row.  A CTA-wide ring of
// 16-row x 2048-k stages beside the slice's activation fragments; K is
// split into slices only when the fragments of all of K leave no room for a
// ring of 4 stages (then 3).
struct MmaPlan {
    bool ok = false;
    int TKC = 0, splits = 1, nks = 0, nrb = 0, cps = 0, grid = 0, stages = 0;
    int cls = kCls128, sz = kSzConst, szw = 0;
    size_t smem = 0, ws = 0;
};

MmaPlan plan_mma(int M, int N, int K, int cls, int sz, int szw, const DeviceInfo& di) {
    MmaPlan p;
    p.cls = cls;
    p.sz = sz;
    p.szw = szw;
    const int nk_total = (K + kMK - 1) / kMK;
    const size_t cap = static_cast<size_t>(di.max_smem_optin);
    // the fewest K slices whose activation fragments leave room for a ring
    // of at least 4 stages (deeper rings first, up to 8), else 3
    for (int min_st : {4, 3}) {
        for (int splits = 1; splits <= nk_total; ++splits) {
            const int nks = (nk_total + splits - 1) / splits;
            int st = 0;
            for (int c = 8; c >= min_st; --c)
                if (gemv_mma_smem_bytes(M, nks * kMK, c, sz, szw) <= cap) {
                    st = c;
                    break;
                }
            if (st == 0) continue;
            p.splits = (nk_total + nks - 1) / nks;
            p.nks = nks;
            p.stages = st;
            break;
        }
        if (p.stages) break;
    }
    if (p.stages == 0) return p;
    p.TKC = p.nks * kMK;
    p.nrb = (N + kMR - 1) / kMR;
    // CTAs per slice: all the SMs, but at least one row block each
    p.cps = std::max(1, std::min(di.sms / p.splits, p.nrb));
    p.grid = p.splits * p.cps;
    p.smem = gemv_mma_smem_bytes(M, p.TKC, p.stages, sz, szw);
    p.ws = p.splits > 1 ? static_cast<size_t>(p.splits) * M * N * sizeof(float) : 0;
    p.ok = true;
    return p;
}

bool mma_eligible(int K, const Meta& meta) { return K % 32 == 0 && (meta.G == 1 || meta.g % 32 == 0); }

// Which packed words a lane holds (WordClass): every k block of one mma
// step must lie in one group.
int mma_cls(const Meta& meta) {
    if (meta.G == 1 || meta.g % 128 == 0) return kCls128;
    return meta.g % 64 == 0 ? kCls64 : kCls32;
}

// How the tensor-pipe GEMV fetches scales and zeros (SzKind) and the width
// that goes with it.
int mma_sz_kind(const Meta& meta) {
    if (meta.sz_row == 0) return kSzConst;
    if (meta.G == 1) return kSzTma1d;
    if (meta.G % 8 == 0 && gemv_mma_sz_box(meta.g) <= 256) return kSzTma2d;
    return kSzCopy;
}
int mma_szw(const Meta& meta, int sz) {
    return sz == kSzTma2d ? gemv_mma_sz_box(meta.g) : sz == kSzCopy ? gemv_mma_sz_words(meta.g) : 0;
}

// group of k = (k * mul) >> shift for 0 <= k < 2^31: with l = ceil(log2 g)
// and mul = floor(2^(31 + l) / g) + 1, k * mul / 2^(31 + l) exceeds k / g
// by less than 2^-l <= 1 / g, so the floor is exact.
void group_magic(int g, unsigned long long* mul, int* shift) {
    int l = 0;
    while ((1ll << l) < g) ++l;
    *shift = 31 + l;
    *mul = (1ull << (31 + l)) / static_cast<unsigned long long>(g) + 1ull;
}

// Int8 tensor-pipe forward GEMV (gemv_q8_kernel): K % 32 == 0 and the
// group length a multiple of 128, or one group per row.  The ring is as deep
// as shared memory allows (up to 8 stages); K is split into slices only to
// give every SM work when there are fewer row blocks than SMs.
struct Q8Plan {
    bool ok = false;
    int TKC = 0, splits = 1, nks = 0, nrb = 0, cps = 0, grid = 0, stages = 0;
    int sz = kSzConst, szw = 0;
    size_t smem = 0, ws = 0;
};

Q8Plan plan_q8(int M, int N, int K, int sz, int szw, const DeviceInfo& di) {
    Q8Plan p;
    p.sz = sz;
    p.szw = szw;
    const size_t cap = static_cast<size_t>(di.max_smem_optin);
    for (int c = 8; c >= 2; --c)
        if (gemv_q8_smem_bytes(c, sz, szw) <= cap) {
            p.stages = c;
            break;
        }
    if (p.stages == 0) return p;
    const int nk_total = (K + kMK - 1) / kMK;
    p.nrb = (N + kMR - 1) / kMR;
    int splits = 1;
    if (2 * p.nrb <= di.sms) splits = std::min(nk_total, std::max(1, di.sms / p.nrb));
    p.nks = (nk_total + splits - 1) / splits;
    p.splits = (nk_total + p.nks - 1) / p.nks;
    p.TKC = p.nks * kMK;
    p.cps = std::max(1, std::min(di.sms / p.splits, p.nrb));
    p.grid = p.splits * p.cps;
    p.smem = gemv_q8_smem_bytes(p.stages, sz, szw);
    p.ws = p.splits > 1 ? static_cast<size_t>(p.splits) * M * N * sizeof(float) : 0;
    p.ok = true;
    return p;
}

bool q8_eligible(int K, const Meta& meta) { return K % 32 == 0 && (meta.G == 1 || meta.g % 128 == 0); }

size_t gemv_workspace(int M, int N, int K, int transposed, int sms) {
    if (transposed) {
        size_t ws = plan_t(M, N, K, sms).ws;
        if (K % 32 == 0)
            for (int kw : {64, 128})
                ws = std::max(ws, plan_t_mma(M, N, K, kw, sms, device_info(current_device()).max_smem_optin).ws);
        return ws;
    }
    if (K % 32 != 0) return 0;
    // the group length sets the stage size, and so possibly the split:
    // cover every choice a group length of 32 .. K can make
    DeviceInfo di = device_info(current_device());
    di.sms = sms;
    size_t ws = plan_q8(M, N, K, kSzConst, 0, di).ws;
    for (int sz : {kSzConst, kSzTma1d}) {
        const MmaPlan q = plan_mma(M, N, K, kCls128, sz, 0, di);
        if (q.ok) ws = std::max(ws, q.ws);
    }
    for (int szw = 8; szw <= 64; szw += 8) {
        const MmaPlan q = plan_mma(M, N, K, kCls128, kSzTma2d, szw, di);
        if (q.ok) ws = std::max(ws, q.ws);
    }
    for (int szw = gemv_mma_sz_words(K); szw <= gemv_mma_sz_words(32); ++szw) {
        const MmaPlan q = plan_mma(M, N, K, kCls128, kSzCopy, szw, di);
        if (q.ok) ws = std::max(ws, q.ws);
    }
    return ws;
}

// The GEMV is always launched as a programmatic dependent of the work just
// before it: its prologue overlaps that work's tail, and it waits for that
// work before reading any input.
template <int M, int CLS, int SZ, bool FZ>
w4_status launch_gemv_mma_k(const MmaPlan& p, const CUtensorMap& wm, const CUtensorMap& sm,
                            const CUtensorMap& zm, const GemvMmaArgs& a, cudaStream_t st) {
    auto* fn = gemv_mma_kernel<M, CLS, SZ, FZ>;
    if (ensure_smem(reinterpret_cast<const void*>(fn), p.smem) != cudaSuccess) return W4_ERR_CUDA;
    launch_pdl(fn, dim3(p.grid), dim3(kMThreads), p.smem, st, wm, sm, zm, a);
    return launch_status();
}

template <int M, int CLS, bool FZ>
w4_status launch_gemv_mma_c(const MmaPlan& p, const CUtensorMap& wm, const CUtensorMap& sm,
                            const CUtensorMap& zm, const GemvMmaArgs& a, cudaStream_t st) {
    switch (p.sz) {
        case kSzConst: return launch_gemv_mma_k<M, CLS, kSzConst, FZ>(p, wm, sm, zm, a, st);
        case kSzTma2d: return launch_gemv_mma_k<M, CLS, kSzTma2d, FZ>(p, wm, sm, zm, a, st);
        case kSzTma1d: return launch_gemv_mma_k<M, CLS, kSzTma1d, FZ>(p, wm, sm, zm, a, st);
        default: return launch_gemv_mma_k<M, CLS, kSzCopy, FZ>(p, wm, sm, zm, a, st);
    }
}

template <int M, bool FZ>
w4_status launch_gemv_mma_m(const MmaPlan& p, const CUtensorMap& wm, const CUtensorMap& sm,
                            const CUtensorMap& zm, const GemvMmaArgs& a, cudaStream_t st) {
    // group lengths that are a multiple of 128 run the int8 kernel
    if (p.cls == kCls64) return launch_gemv_mma_c<M, kCls64, FZ>(p, wm, sm, zm, a, st);
    return launch_gemv_mma_c<M, kCls32, FZ>(p, wm, sm, zm, a, st);
}

w4_status run_gemv_mma(const MmaPlan& p, int M, int N, int K, const void* A, const uint32_t* packed,
                       const void* S, const void* Z, const Meta& meta, const void* bias, void* Y, void* ws,
                       size_t ws_bytes, cudaStream_t st) {
    if (p.ws > ws_bytes || (p.ws > 0 && ws == nullptr)) return W4_ERR_WORKSPACE;
    if (ws && !aligned16(ws)) return W4_ERR_ALIGNMENT;
    float* partial = p.splits > 1 ? static_cast<float*>(ws) : nullptr;
    CUtensorMap wm, sm, zm;
    std::memset(&sm, 0, sizeof sm);
    std::memset(&zm, 0, sizeof zm);
    bool ok = make_map_2d(&wm, packed, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, N, K / 8, kMR, kMK / 8, 0);
    if (p.sz == kSzTma2d) {
        ok = ok && make_map_2d(&sm, S, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, meta.G, kMR, p.szw, 0) &&
             make_map_2d(&zm, Z, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, meta.G, kMR, p.szw, 0);
    } else if (p.sz == kSzTma1d) {
        ok = ok && make_map_row(&sm, S, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, kMR) &&
             make_map_row(&zm, Z, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, kMR);
    }
    if (!ok) return W4_ERR_CUDA;
    GemvMmaArgs a;
    a.X = static_cast<const uint16_t*>(A);
    a.S = static_cast<const __half*>(S);
    a.Z = static_cast<const __half*>(Z);
    a.bias = static_cast<const uint16_t*>(bias);
    a.Y = static_cast<uint16_t*>(Y);
    a.partial = partial;
    a.N = N;
    a.K = K;
    a.g = meta.g;
    a.G = meta.G;
    a.sz_row = meta.sz_row;
    a.fmt = meta.fmt;
    group_magic(meta.g, &a.gmul, &a.gshift);
    a.TKC = p.TKC;
    a.splits = p.splits;
    a.nks = p.nks;
    a.nrb = p.nrb;
    a.cps = p.cps;
    a.stages = p.stages;
    a.szw = p.szw;
    a.sz_total = meta.sz_row ? static_cast<long long>(N) * meta.sz_row : 1;
    w4_status s = W4_OK;
    const bool fz = (meta.fmt & kFmtZeroFloat) != 0;
    switch (M) {
        case 1: s = fz ? launch_gemv_mma_m<1, true>(p, wm, sm, zm, a, st) : launch_gemv_mma_m<1, false>(p, wm, sm, zm, a, st); break;
        case 2: s = fz ? launch_gemv_mma_m<2, true>(p, wm, sm, zm, a, st) : launch_gemv_mma_m<2, false>(p, wm, sm, zm, a, st); break;
        case 3: s = fz ? launch_gemv_mma_m<3, true>(p, wm, sm, zm, a, st) : launch_gemv_mma_m<3, false>(p, wm, sm, zm, a, st); break;
        case 4: s = fz ? launch_gemv_mma_m<4, true>(p, wm, sm, zm, a, st) : launch_gemv_mma_m<4, false>(p, wm, sm, zm, a, st); break;
        default: return W4_ERR_INVALID_ARG;
    }
    if (s != W4_OK) return s;
    if (p.splits > 1) {
        const DeviceInfo di = device_info(current_device());
        const long long total = static_cast<long long>(M) * N;
        const int blocks = static_cast<int>(std::min<long long>((total + kFinOut - 1) / kFinOut, di.sms * 16));
        launch_pdl(splits_finalize_kernel, dim3(blocks), dim3(256), 0, st, static_cast<const float*>(partial),
                   p.splits, M, N, static_cast<const uint16_t*>(bias), static_cast<uint16_t*>(Y));
        return launch_status();
    }
    return W4_OK;
}

template <int M, int SZ, bool FZ>
w4_status launch_q8_k(const Q8Plan& p, const CUtensorMap& wm, const CUtensorMap& sm, const CUtensorMap& zm,
                      const GemvQ8Args& a, cudaStream_t st) {
    auto* fn = gemv_q8_kernel<M, SZ, FZ>;
    if (ensure_smem(reinterpret_cast<const void*>(fn), p.smem) != cudaSuccess) return W4_ERR_CUDA;
    launch_pdl(fn, dim3(p.grid), dim3(kQThreads), p.smem, st, wm, sm, zm, a);
    return launch_status();
}

template <int M, bool FZ>
w4_status launch_q8_m(const Q8Plan& p, const CUtensorMap& wm, const CUtensorMap& sm, const CUtensorMap& zm,
                      const GemvQ8Args& a, cudaStream_t st) {
    switch (p.sz) {
        case kSzConst: return launch_q8_k<M, kSzConst, FZ>(p, wm, sm, zm, a, st);
        case kSzTma2d: return launch_q8_k<M, kSzTma2d, FZ>(p, wm, sm, zm, a, st);
        case kSzTma1d: return launch_q8_k<M, kSzTma1d, FZ>(p, wm, sm, zm, a, st);
        default: return launch_q8_k<M, kSzCopy, FZ>(p, wm, sm, zm, a, st);
    }
}

w4_status run_gemv_q8(const Q8Plan& p, int M, int N, int K, const void* A, const uint32_t* packed, const void* S,
                      const void* Z, const Meta& meta, const void* bias, void* Y, void* ws, size_t ws_bytes,
                      cudaStream_t st) {
    if (p.ws > ws_bytes || (p.ws > 0 && ws == nullptr)) return W4_ERR_WORKSPACE;
    if (ws && !aligned16(ws)) return W4_ERR_ALIGNMENT;
    float* partial = p.splits > 1 ? static_cast<float*>(ws) : nullptr;
    CUtensorMap wm, sm, zm;
    std::memset(&sm, 0, sizeof sm);
    std::memset(&zm, 0, sizeof zm);
    bool ok = make_map_2d(&wm, packed, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, N, K / 8, kMR, kMK / 8, 0);
    if (p.sz == kSzTma2d) {
        ok = ok && make_map_2d(&sm, S, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, meta.G, kMR, p.szw, 0) &&
             make_map_2d(&zm, Z, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, meta.G, kMR, p.szw, 0);
    } else if (p.sz == kSzTma1d) {
        ok = ok && make_map_row(&sm, S, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, kMR) &&
             make_map_row(&zm, Z, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, kMR);
    }
    if (!ok) return W4_ERR_CUDA;
    GemvQ8Args a;
    a.X = static_cast<const uint16_t*>(A);
    a.S = static_cast<const __half*>(S);
    a.Z = static_cast<const __half*>(Z);
    a.bias = static_cast<const uint16_t*>(bias);
    a.Y = static_cast<uint16_t*>(Y);
    a.partial = partial;
    a.N = N;
    a.K = K;
    a.g = meta.g;
    a.G = meta.G;
    a.sz_row = meta.sz_row;
    a.fmt = meta.fmt;
    group_magic(meta.g, &a.gmul, &a.gshift);
    a.TKC = p.TKC;
    a.splits = p.splits;
    a.nks = p.nks;
    a.nrb = p.nrb;
    a.cps = p.cps;
    a.stages = p.stages;
    a.szw = p.szw;
    a.sz_total = meta.sz_row ? static_cast<long long>(N) * meta.sz_row : 1;
    w4_status s = W4_OK;
    const bool fz = (meta.fmt & kFmtZeroFloat) != 0;
    switch (M) {
        case 1: s = fz ? launch_q8_m<1, true>(p, wm, sm, zm, a, st) : launch_q8_m<1, false>(p, wm, sm, zm, a, st); break;
        case 2: s = fz ? launch_q8_m<2, true>(p, wm, sm, zm, a, st) : launch_q8_m<2, false>(p, wm, sm, zm, a, st); break;
        case 3: s = fz ? launch_q8_m<3, true>(p, wm, sm, zm, a, st) : launch_q8_m<3, false>(p, wm, sm, zm, a, st); break;
        case 4: s = fz ? launch_q8_m<4, true>(p, wm, sm, zm, a, st) : launch_q8_m<4, false>(p, wm, sm, zm, a, st); break;
        default: return W4_ERR_INVALID_ARG;
    }
    if (s != W4_OK) return s;
    if (p.splits > 1) {
        const DeviceInfo di = device_info(current_device());
        const long long total = static_cast<long long>(M) * N;
        const int blocks = static_cast<int>(std::min<long long>((total + kFinOut - 1) / kFinOut, di.sms * 16));
        launch_pdl(splits_finalize_kernel, dim3(blocks), dim3(256), 0, st, static_cast<const float*>(partial),
                   p.splits, M, N, static_cast<const uint16_t*>(bias), static_cast<uint16_t*>(Y));
        return launch_status();
    }
    return W4_OK;
}

w4_status run_gemv_fwd(const void* A, int M, int N, int K, const uint32_t* packed, const void* S,
                       const void* Z, const Meta& meta, const void* bias, void* Y, void* ws,
                       size_t ws_bytes, cudaStream_t st) {
    const DeviceInfo di = device_info(current_device());
    if (q8_eligible(K, meta)) {
        const int sz = mma_sz_kind(meta);
        const Q8Plan qp = plan_q8(M, N, K, sz, mma_szw(meta, sz), di);
        if (qp.ok) return run_gemv_q8(qp, M, N, K, A, packed, S, Z, meta, bias, Y, ws, ws_bytes, st);
    }
    if (mma_eligible(K, meta)) {
        const int sz = mma_sz_kind(meta);
        const MmaPlan mp = plan_mma(M, N, K, mma_cls(meta), sz, mma_szw(meta, sz), di);
        if (mp.ok) return run_gemv_mma(mp, M, N, K, A, packed, S, Z, meta, bias, Y, ws, ws_bytes, st);
    }
    // K or the group length not a multiple of 32: one warp per output row
    GemvFwdArgs a;
    a.X = static_cast<const uint16_t*>(A);
    a.S = static_cast<const __half*>(S);
    a.Z = static_cast<const __half*>(Z);
    a.bias = static_cast<const uint16_t*>(bias);
    a.Y = static_cast<uint16_t*>(Y);
    a.N = N;
    a.K = K;
    a.g = meta.g;
    a.G = meta.G;
    a.sz_row = meta.sz_row;
    a.fmt = meta.fmt;
    const int blocks = static_cast<int>((static_cast<long long>(N) * 32 + 255) / 256);
    switch (M) {
        case 1: gemv_fwd_simple_kernel<1><<<blocks, 256, 0, st>>>(a, packed); break;
        case 2: gemv_fwd_simple_kernel<2><<<blocks, 256, 0, st>>>(a, packed); break;
        case 3: gemv_fwd_simple_kernel<3><<<blocks, 256, 0, st>>>(a, packed); break;
        case 4: gemv_fwd_simple_kernel<4><<<blocks, 256, 0, st>>>(a, packed); break;
        default: return W4_ERR_INVALID_ARG;
    }
    return launch_status();
}

template <int M, int KW, int SZ, bool FZ>
w4_status launch_t_mma_k(const TMmaPlan& p, const CUtensorMap& wm, const CUtensorMap& sm, const CUtensorMap& zm,
                         const GemvTMmaArgs& a, cudaStream_t st) {
    auto* fn = gemv_t_mma_kernel<M, KW, SZ, FZ>;
    if (ensure_smem(reinterpret_cast<const void*>(fn), p.smem) != cudaSuccess) return W4_ERR_CUDA;
    launch_pdl(fn, dim3(p.grid), dim3(kTMThreads), p.smem, st, wm, sm, zm, a);
    return launch_status();
}

template <int M, int KW, bool FZ>
w4_status launch_t_mma_kw(const TMmaPlan& p, int sz, const CUtensorMap& wm, const CUtensorMap& sm,
                          const CUtensorMap& zm, const GemvTMmaArgs& a, cudaStream_t st) {
    switch (sz) {
        case kSzConst: return launch_t_mma_k<M, KW, kSzConst, FZ>(p, wm, sm, zm, a, st);
        case kSzTma1d: return launch_t_mma_k<M, KW, kSzTma1d, FZ>(p, wm, sm, zm, a, st);
        default: return launch_t_mma_k<M, KW, kSzTma2d, FZ>(p, wm, sm, zm, a, st);
    }
}

template <int M, bool FZ>
w4_status launch_t_mma_m(const TMmaPlan& p, int sz, const CUtensorMap& wm, const CUtensorMap& sm,
                         const CUtensorMap& zm, const GemvTMmaArgs& a, cudaStream_t st) {
    // M = 3, 4 always take KW = 64 (two column sets)
    if (M <= 2 && p.KW == 128) return launch_t_mma_kw<M, (M <= 2 ? 128 : 64), FZ>(p, sz, wm, sm, zm, a, st);
    return launch_t_mma_kw<M, 64, FZ>(p, sz, wm, sm, zm, a, st);
}

w4_status run_gemv_t_mma(const TMmaPlan& p, int sz, int M, int N, int K, const void* A, const uint32_t* packed,
                         const void* S, const void* Z, const Meta& meta, const void* bias, void* Y, void* ws,
                         size_t ws_bytes, cudaStream_t st) {
    if (p.ws > ws_bytes || (p.ws > 0 && ws == nullptr)) return W4_ERR_WORKSPACE;
    CUtensorMap wm, sm, zm;
    std::memset(&sm, 0, sizeof sm);
    std::memset(&zm, 0, sizeof zm);
    // packed rows as K / 16 8-byte elements: boxes of 32 rows x (strip + 16) bytes
    bool ok = make_map_2d(&wm, packed, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, N, K / 16, kTMRows, tm_pitch(p.KW) / 8, 0);
    if (sz == kSzTma2d)
        ok = ok && make_map_2d(&sm, S, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, meta.G, kTMRows, 16, 0) &&
             make_map_2d(&zm, Z, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, meta.G, kTMRows, 16, 0);
    else if (sz == kSzTma1d)
        ok = ok && make_map_row(&sm, S, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, kTMRows) &&
             make_map_row(&zm, Z, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, kTMRows);
    if (!ok) return W4_ERR_CUDA;
    GemvTMmaArgs a;
    a.dY = static_cast<const uint16_t*>(A);
    a.packed = packed;
    a.S = static_cast<const __half*>(S);
    a.Z = static_cast<const __half*>(Z);
    a.bias = static_cast<const uint16_t*>(bias);
    a.dX = static_cast<uint16_t*>(Y);
    a.partial = static_cast<float*>(ws);
    a.N = N;
    a.K = K;
    a.g = meta.g;
    a.G = meta.G;
    a.sz_row = meta.sz_row;
    a.fmt = meta.fmt;
    a.strips = p.strips;
    a.splits = p.splits;
    a.rows_per_split = p.rows_per_split;
    a.stages = p.stages;
    w4_status s = W4_OK;
    const bool fz = (meta.fmt & kFmtZeroFloat) != 0;
    switch (M) {
        case 1: s = fz ? launch_t_mma_m<1, true>(p, sz, wm, sm, zm, a, st) : launch_t_mma_m<1, false>(p, sz, wm, sm, zm, a, st); break;
        case 2: s = fz ? launch_t_mma_m<2, true>(p, sz, wm, sm, zm, a, st) : launch_t_mma_m<2, false>(p, sz, wm, sm, zm, a, st); break;
        case 3: s = fz ? launch_t_mma_m<3, true>(p, sz, wm, sm, zm, a, st) : launch_t_mma_m<3, false>(p, sz, wm, sm, zm, a, st); break;
        case 4: s = fz ? launch_t_mma_m<4, true>(p, sz, wm, sm, zm, a, st) : launch_t_mma_m<4, false>(p, sz, wm, sm, zm, a, st); break;
        default: return W4_ERR_INVALID_ARG;
    }
    if (s != W4_OK) return s;
    if (p.splits > 1) {
        // a programmatic dependent: its launch overlaps the split kernel,
        // whose partials it waits for
        const DeviceInfo di = device_info(current_device());
        const long long total4 = static_cast<long long>(M) * K / 4;     // K % 32 == 0
        const int blocks = static_cast<int>(std::min<long long>((total4 + kFin4Cols - 1) / kFin4Cols, di.sms * 8));
        launch_pdl(splits_finalize_vec4_kernel, dim3(blocks), dim3(256), 0, st,
                   static_cast<const float*>(a.partial), p.splits, M, K, a.bias, a.dX);
        return launch_status();
    }
    return W4_OK;
}

w4_status run_gemv_t(const void* A, int M, int N, int K, const uint32_t* packed, const void* S,
                     const void* Z, const Meta& meta, const void* bias, void* Y, void* ws,
                     size_t ws_bytes, cudaStream_t st) {
    const DeviceInfo di = device_info(current_device());
    if (t_mma_eligible(K, meta)) {
        const int sz = meta.sz_row == 0 ? kSzConst : (meta.G == 1 ? kSzTma1d : kSzTma2d);
        const TMmaPlan mp = plan_t_mma(M, N, K, t_mma_kw(M, meta), di.sms, di.max_smem_optin);
        if (mp.ok) return run_gemv_t_mma(mp, sz, M, N, K, A, packed, S, Z, meta, bias, Y, ws, ws_bytes, st);
    }
    const TPlan p = plan_t(M, N, K, di.sms);
    if (p.ws > ws_bytes || (p.ws > 0 && ws == nullptr)) return W4_ERR_WORKSPACE;
    GemvTArgs a;
    a.dY = static_cast<const uint16_t*>(A);
    a.packed = packed;
    a.S = static_cast<const __half*>(S);
    a.Z = static_cast<const __half*>(Z);
    a.bias = static_cast<const uint16_t*>(bias);
    a.dX = static_cast<uint16_t*>(Y);
    a.partial = static_cast<float*>(ws);
    a.N = N;
    a.K = K;
    a.g = meta.g;
    a.G = meta.G;
    a.sz_row = meta.sz_row;
    a.fmt = meta.fmt;
    a.rows_per_split = p.rows_per_split;
    a.splits = p.splits;
    const dim3 grid((K / 8 + kGemvTWordsPerCta - 1) / kGemvTWordsPerCta, p.splits);
    switch (M) {
        case 1: gemv_t_kernel<1><<<grid, kGemvTThreads, 0, st>>>(a); break;
        case 2: gemv_t_kernel<2><<<grid, kGemvTThreads, 0, st>>>(a); break;
        case 3: gemv_t_kernel<3><<<grid, kGemvTThreads, 0, st>>>(a); break;
        case 4: gemv_t_kernel<4><<<grid, kGemvTThreads, 0, st>>>(a); break;
    }
    w4_status s = launch_status();
    if (s != W4_OK) return s;
    if (p.splits > 1) {
        const long long total = static_cast<long long>(M) * K;
        const int blocks = static_cast<int>(std::min<long long>((total + kFinOut - 1) / kFinOut, di.sms * 16));
        splits_finalize_kernel<<<blocks, 256, 0, st>>>(a.partial, p.splits, M, K, a.bias, a.dX);
        return launch_status();
    }
    return W4_OK;
}

// Common argument checks of the matmul entry points, in the documented order.
w4_status check_matmul(const void* A, int M, int N, int K, const uint32_t* packed, const void* S,
                       const void* Z, int mode, int group_size, const void* bias, void* Y,
                       Meta* meta) {
    if (M <= 0 || N <= 0 || K <= 0) return W4_ERR_INVALID_ARG;
    if (K % 8 != 0) return W4_ERR_INVALID_ARG;
    w4_status s = check_mode(K, mode, group_size, meta);
    if (s != W4_OK) return s;
    if (!A || !packed || !S || !Z || !Y) return W4_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(packed) || !aligned16(S) || !aligned16(Z) || !aligned16(Y) ||
        (bias && !aligned16(bias)))
        return W4_ERR_ALIGNMENT;
    return W4_OK;
}

w4_status run_gemv(const void* A, int M, int N, int K, const uint32_t* packed, const void* S,
                   const void* Z, const Meta& meta, const void* bias, int transposed, void* Y,
                   void* ws, size_t ws_bytes, cudaStream_t st) {
    return transposed ? run_gemv_t(A, M, N, K, packed, S, Z, meta, bias, Y, ws, ws_bytes, st)
                      : run_gemv_fwd(A, M, N, K, packed, S, Z, meta, bias, Y, ws, ws_bytes, st);
}


// ---------------------------------------------------------- tensor-core GEMM
int tc_pick_bn(int M) {
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

// Work split of the persistent GEMM.  With T tiles on P SMs, T / P whole
// waves run as whole tiles; the R = T mod P tiles of a last partial wave
// (all tiles, when T < P) are cut into S slices of their k-blocks when that
// pays: the tail then takes ceil(R S / P) / S of a tile's time instead of a
// whole one, against the cost of writing and re-reading R S fp32 partial
// tiles plus a finalize launch; S maximizes the difference.  Slices keep at
// least 4 k-blocks.
struct TcPlan {
    int BN = 0, tiles_m = 0, tiles = 0, F = 0, S = 1, grid = 0;
    size_t ws = 0;
};

TcPlan plan_tc(int M, int N, int K, int transposed, int sms) {
    TcPlan p;
    p.BN = tc_pick_bn(M);
    const int L_out = transposed ? K : N;
    const int red = transposed ? N : K;
    const int num_kb = (red + kTcBK - 1) / kTcBK;
    p.tiles_m = (M + p.BN - 1) / p.BN;
    const long long tiles = static_cast<long long>(p.tiles_m) * ((L_out + kTcBM - 1) / kTcBM);
    p.tiles = static_cast<int>(std::min<long long>(tiles, 1ll << 30));
    const int P = std::max(1, sms);
    const int R = p.tiles % P;
    p.F = p.tiles;
    if (R > 0) {
        // a tile's time in microseconds, roughly: the slower of its tensor
        // work (a 64-k block of 128 x BN takes ~0.75 us per 256 tokens at the
        // rates this kernel reaches) and its bytes (128 packed rows and BN
        // activation rows over the reduction) at one SM's share of HBM
        // (~40 GB/s); small tiles are bound by the latter
        const double bytes = static_cast<double>(red) * (kTcBM / 2.0 + 2.0 * p.BN);
        const double tile_us = std::max(num_kb * (p.BN / 256.0) * 0.75, bytes / 40.0e3);
        double best = 0.0;
        int bestS = 1;
        for (int S = 2; S <= std::min(16, num_kb / 4); ++S) {
            const double tail = static_cast<double>((static_cast<long long>(R) * S + P - 1) / P) / S;
            // the partials are written and read back through L2 (~8 TB/s)
            const double cost = 3.0 + 2.0 * R * S * p.BN * kTcBM * 4 / 8.0e6;   // us
            const double gain = (1.0 - tail) * tile_us - cost;
            if (gain > best + 1e-9) {
                best = gain;
                bestS = S;
            }
        }
        if (bestS > 1) {
            p.S = bestS;
            p.F = p.tiles - R;
        }
    }
    const long long units = p.F + static_cast<long long>(p.tiles - p.F) * p.S;
    p.grid = static_cast<int>(std::min<long long>(units, P));
    p.ws = static_cast<size_t>(p.tiles - p.F) * p.S * p.BN * kTcBM * sizeof(float);
    return p;
}

size_t gemm_tc_workspace_bytes(int M, int N, int K, int transposed, int sms) {
    if (K % 32 != 0 || (transposed && N % 8 != 0)) return 0;   // the plain kernel needs none
    return plan_tc(M, N, K, transposed, sms).ws;
}

template <bool TR, int BN, bool PWG, bool FZ>
w4_status launch_tc(const CUtensorMap& pm, const CUtensorMap& bm, const CUtensorMap& sm, const CUtensorMap& zm,
                    const TcArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    const void* fn = reinterpret_cast<const void*>(gemm_tc_kernel<TR, BN, PWG, FZ>);
    if (ensure_smem(fn, smem) != cudaSuccess) return W4_ERR_CUDA;
    gemm_tc_kernel<TR, BN, PWG, FZ><<<grid, kTcThreads, smem, st>>>(pm, bm, sm, zm, a);
    return launch_status();
}

template <bool TR, bool PWG, bool FZ>
w4_status launch_tc_bn(int BN, const CUtensorMap* m, const TcArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    switch (BN) {
        case 16: return launch_tc<TR, 16, PWG, FZ>(m[0], m[1], m[2], m[3], a, grid, smem, st);
        case 32: return launch_tc<TR, 32, PWG, FZ>(m[0], m[1], m[2], m[3], a, grid, smem, st);
        case 64: return launch_tc<TR, 64, PWG, FZ>(m[0], m[1], m[2], m[3], a, grid, smem, st);
        case 128: return launch_tc<TR, 128, PWG, FZ>(m[0], m[1], m[2], m[3], a, grid, smem, st);
        default: return launch_tc<TR, 256, PWG, FZ>(m[0], m[1], m[2], m[3], a, grid, smem, st);
    }
}

template <bool TR, bool PWG>
w4_status launch_tc_fz(bool fz, int BN, const CUtensorMap* m, const TcArgs& a, dim3 grid, size_t smem,
                       cudaStream_t st) {
    return fz ? launch_tc_bn<TR, PWG, true>(BN, m, a, grid, smem, st)
              : launch_tc_bn<TR, PWG, false>(BN, m, a, grid, smem, st);
}

// Shapes whose rows TMA cannot stream: the plain CUDA-core kernel.
w4_status run_gemm_simple(const TcProblem& p, cudaStream_t st) {
    GemmSimpleArgs a;
    a.A = static_cast<const uint16_t*>(p.A);
    a.packed = p.packed;
    a.S = static_cast<const __half*>(p.S);
    a.Z = static_cast<const __half*>(p.Z);
    a.bias = static_cast<const uint16_t*>(p.bias);
    a.Y = static_cast<uint16_t*>(p.Y);
    a.M = p.M;
    a.N = p.N;
    a.K = p.K;
    a.g = p.g;
    a.G = p.G;
    a.sz_row = p.sz_row;
    a.fmt = p.fmt;
    const int L = p.transposed ? p.K : p.N;
    const dim3 grid((L + kGsTile - 1) / kGsTile, (p.M + kGsTile - 1) / kGsTile);
    if (p.transposed)
        gemm_simple_kernel<true><<<grid, 256, 0, st>>>(a);
    else
        gemm_simple_kernel<false><<<grid, 256, 0, st>>>(a);
    return launch_status();
}

w4_status run_gemm_tc(const TcProblem& p, void* ws, size_t ws_bytes, cudaStream_t st) {
    // packed rows (and dY rows when transposed) must be 16-byte strided for TMA
    if (p.K % 32 != 0 || (p.transposed && p.N % 8 != 0)) return run_gemm_simple(p, st);
    const DeviceInfo di = device_info(current_device());
    const TcPlan plan = plan_tc(p.M, p.N, p.K, p.transposed, di.sms);
    if (plan.ws > ws_bytes || (plan.ws > 0 && ws == nullptr)) return W4_ERR_WORKSPACE;
    const int BN = plan.BN;
    const bool tr = p.transposed != 0;
    // scales and zeros ride on each stage as 8-group TMA boxes when the rows
    // are 16-byte strided and a stage's k range (64, transposed 128) never
    // leaves the box that starts at its first group rounded down to 8
    const int L = tr ? 128 : kTcBK;
    const bool sz_tma = p.G > 1 && p.G % 8 == 0 &&
                        (p.g % L == 0 || (L % p.g == 0 && L / p.g <= 8));
    const int sz_rows = tr ? kTcBK : kTcBM;
    const int stage = tc_stage_bytes(BN) + (sz_tma ? 2 * sz_rows * 16 : 0);
    const size_t fixed = 1024 + 64;
    int stages = static_cast<int>((static_cast<size_t>(di.max_smem_optin) - fixed - 64) / (stage + 32));
    stages = std::min(stages, 8);
    if (stages < 2) return W4_ERR_UNSUPPORTED;
    const size_t smem = fixed + static_cast<size_t>(stages) * stage + static_cast<size_t>(4 * stages + 4) * 8 + 16;
    CUtensorMap maps[4];
    std::memset(maps, 0, sizeof maps);
    CUtensorMap& pm = maps[0];
    CUtensorMap& bm = maps[1];
    // packed weights [N, K/8] uint32: box 8 words x 128 rows (forward) or
    // 16 words x 64 rows (transposed); activations [M, K] or dY [M, N] bf16,
    // box 64 x BN with the 128-byte swizzle the MMA descriptors expect
    bool ok = tr ? make_map_2d(&pm, p.packed, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, p.N, p.K / 8, 64, 16, 0)
                 : make_map_2d(&pm, p.packed, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, p.N, p.K / 8, 128, 8, 0);
    ok = ok && make_map_2d(&bm, p.A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.M, tr ? p.N : p.K, BN, 64, 128);
    if (sz_tma)
        ok = ok && make_map_2d(&maps[2], p.S, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.N, p.G, sz_rows, 8, 0) &&
             make_map_2d(&maps[3], p.Z, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.N, p.G, sz_rows, 8, 0);
    if (!ok) return W4_ERR_CUDA;
    TcArgs a;
    a.S = static_cast<const __half*>(p.S);
    a.Z = static_cast<const __half*>(p.Z);
    a.bias = static_cast<const uint16_t*>(p.bias);
    a.Y = static_cast<uint16_t*>(p.Y);
    a.M = p.M;
    a.N = p.N;
    a.K = p.K;
    a.g = p.g;
    a.G = p.G;
    a.sz_row = p.sz_row;
    a.fmt = p.fmt;
    a.stages = stages;
    a.stage_bytes = stage;
    a.sz_tma = sz_tma ? 1 : 0;
    a.part = static_cast<float*>(ws);
    a.F = plan.F;
    a.nslice = plan.S;
    const int L_out = tr ? p.K : p.N;
    if (static_cast<long long>(p.M + BN - 1) / BN * ((L_out + kTcBM - 1) / kTcBM) > (1ll << 30))
        return W4_ERR_UNSUPPORTED;
    // persistent: one CTA per SM (or per work unit, when there are fewer)
    const dim3 grid(static_cast<unsigned>(plan.grid));
    const bool pwg = (p.g % 32) != 0;
    const bool fz = (p.fmt & kFmtZeroFloat) != 0;
    w4_status s = tr ? (pwg ? launch_tc_fz<true, true>(fz, BN, maps, a, grid, smem, st)
                            : launch_tc_fz<true, false>(fz, BN, maps, a, grid, smem, st))
                     : (pwg ? launch_tc_fz<false, true>(fz, BN, maps, a, grid, smem, st)
                            : launch_tc_fz<false, false>(fz, BN, maps, a, grid, smem, st));
    if (s != W4_OK || plan.F == plan.tiles) return s;
    const long long threads = static_cast<long long>(plan.tiles - plan.F) * BN * (kTcBM / 4);
    launch_pdl(gemm_tail_finalize_kernel, dim3(static_cast<unsigned>((threads + 255) / 256)), dim3(256), 0, st,
               static_cast<const float*>(a.part), plan.F, plan.S, plan.tiles - plan.F, plan.tiles_m, BN, p.M, L_out,
               a.bias, a.Y);
    return launch_status();
}


// ------------------------------------------------- allocation-free GEMV
// Scratch for w4a16_gemv_noalloc: the forward GEMV's workspace (prepared
// activations, split-K partials) lives in this file-scope array instead of
// a caller workspace.  Every device that loads the library holds one copy
// until the process exits.
constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of the scratch array on the current device.  Host code
// cannot pass &g_noalloc_scratch to a kernel (that name is a host-side
// stand-in), so every call looks the address up with the device current
// (the lookup allocates nothing).  It is not cached: after cudaDeviceReset,
// or a primary context torn down and created again, the module is loaded
// anew and the array may sit at another address.
w4_status noalloc_scratch(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
        g_last_cuda_error = cudaGetLastError();
        return W4_ERR_CUDA;
    }
    *out = p;
    return W4_OK;
}

}  // namespace

extern "C" {

const char* w4_status_string(int status) {
    switch (status) {
        case W4_OK: return "W4_OK";
        case W4_ERR_INVALID_ARG: return "W4_ERR_INVALID_ARG: a size, mode or group size is out of range";
        case W4_ERR_UNSUPPORTED: return "W4_ERR_UNSUPPORTED: valid arguments that no kernel here handles";
        case W4_ERR_ALIGNMENT: return "W4_ERR_ALIGNMENT: a pointer is not 16-byte aligned";
        case W4_ERR_WORKSPACE: return "W4_ERR_WORKSPACE: workspace missing or too small";
        case W4_ERR_CUDA: return "W4_ERR_CUDA: a CUDA call or kernel launch failed";
        case W4_ERR_TIMEOUT: return "W4_ERR_TIMEOUT: a kernel abandoned a bounded wait";
        default: return "unknown w4_status";
    }
}

size_t w4_quantize_workspace_bytes(int N, int K, int mode) {
    (void)N;
    (void)K;
    return (mode & kModeBaseMask) == W4_MODE_GLOBAL ? 1024 * sizeof(float2) : 0;
}

}  // extern "C"

namespace {
// The segmented quantizer with its format flags as a template argument.
template <int LPG, int WPT>
void launch_quantize_segmented(int fmt, int blocks, cudaStream_t st, const uint16_t* w, long long total_words,
                               uint32_t* packed, uint16_t* sc, uint16_t* ze) {
    using w4::kFmtMetaBf16;
    using w4::kFmtZeroFloat;
    switch (fmt & (kFmtZeroFloat | kFmtMetaBf16)) {
        case 0:
            w4::quantize_segmented_kernel<LPG, WPT, 0><<<blocks, 256, 0, st>>>(w, total_words, packed, sc, ze);
            break;
        case kFmtZeroFloat:
            w4::quantize_segmented_kernel<LPG, WPT, kFmtZeroFloat><<<blocks, 256, 0, st>>>(w, total_words, packed,
                                                                                          sc, ze);
            break;
        case kFmtMetaBf16:
            w4::quantize_segmented_kernel<LPG, WPT, kFmtMetaBf16><<<blocks, 256, 0, st>>>(w, total_words, packed,
                                                                                         sc, ze);
            break;
        default:
            w4::quantize_segmented_kernel<LPG, WPT, kFmtZeroFloat | kFmtMetaBf16>
                <<<blocks, 256, 0, st>>>(w, total_words, packed, sc, ze);
    }
}
}  // namespace

extern "C" {

w4_status w4_quantize_pack(const void* W, int N, int K, int mode, int group_size, uint32_t* packed,
                           void* scales, void* zeros, void* workspace, size_t workspace_bytes,
                           void* stream) {
    if (N <= 0 || K <= 0 || K % 8 != 0) return W4_ERR_INVALID_ARG;
    Meta meta;
    w4_status s = check_mode(K, mode, group_size, &meta);
    if (s != W4_OK) return s;
    if (!W || !packed || !scales || !zeros) return W4_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(scales) || !aligned16(zeros))
        return W4_ERR_ALIGNMENT;
    const size_t need = w4_quantize_workspace_bytes(N, K, mode);
    if (workspace_bytes < need || (need > 0 && !workspace)) return W4_ERR_WORKSPACE;
    if (need > 0 && !aligned16(workspace)) return W4_ERR_ALIGNMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (g_debug_checks.load(std::memory_order_relaxed)) {
        // reject NaN / Inf weights before quantizing (synchronizes the stream)
        unsigned int flag = 0;
        if (cudaMemcpyToSymbolAsync(w4::g_nonfinite, &flag, sizeof flag, 0, cudaMemcpyHostToDevice, st) !=
            cudaSuccess)
            return W4_ERR_CUDA;
        const long long n = static_cast<long long>(N) * K;
        const int blocks = static_cast<int>(std::min<long long>((n / 8 + 255) / 256, 1024));
        nonfinite_check_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint16_t*>(W), n);
        s = launch_status();
        if (s != W4_OK) return s;
        if (cudaMemcpyFromSymbolAsync(&flag, w4::g_nonfinite, sizeof flag, 0, cudaMemcpyDeviceToHost, st) !=
                cudaSuccess ||
            cudaStreamSynchronize(st) != cudaSuccess)
            return W4_ERR_CUDA;
        if (flag) return W4_ERR_INVALID_ARG;
    }
    const uint16_t* w = static_cast<const uint16_t*>(W);
    uint16_t* sc = static_cast<uint16_t*>(scales);
    uint16_t* ze = static_cast<uint16_t*>(zeros);
    const int fmt = meta.fmt;
    const long long total_words = static_cast<long long>(N) * (K / 8);
    const DeviceInfo di = device_info(current_device());
    if ((mode & kModeBaseMask) == W4_MODE_GLOBAL) {
        const int blocks = static_cast<int>(
            std::min<long long>(1024, std::min<long long>((total_words + 255) / 256, di.sms * 4)));
        float2* part = static_cast<float2*>(workspace);
        global_minmax_kernel<<<blocks, 256, 0, st>>>(w, total_words, part);
        s = launch_status();
        if (s != W4_OK) return s;
        const int qblocks =
            static_cast<int>(std::min<long long>((total_words + 255) / 256, di.sms * 8));
        global_quantize_kernel<<<qblocks, 256, 0, st>>>(w, total_words, part, blocks, packed, sc, ze, fmt);
        return launch_status();
    }
    // words per group: two words per thread (one for g = 8), lanes of a group
    // reduce with shuffles up to a warp; longer groups take a warp each
    const int lpg = meta.g / 8;
    const int wpt = lpg >= 2 ? 2 : 1;
    const int blocks = static_cast<int>((total_words / wpt + 255) / 256);
    switch (lpg) {
        case 1: launch_quantize_segmented<1, 1>(fmt, blocks, st, w, total_words, packed, sc, ze); break;
        case 2: launch_quantize_segmented<1, 2>(fmt, blocks, st, w, total_words, packed, sc, ze); break;
        case 4: launch_quantize_segmented<2, 2>(fmt, blocks, st, w, total_words, packed, sc, ze); break;
        case 8: launch_quantize_segmented<4, 2>(fmt, blocks, st, w, total_words, packed, sc, ze); break;
        case 16: launch_quantize_segmented<8, 2>(fmt, blocks, st, w, total_words, packed, sc, ze); break;
        case 32: launch_quantize_segmented<16, 2>(fmt, blocks, st, w, total_words, packed, sc, ze); break;
        case 64: launch_quantize_segmented<32, 2>(fmt, blocks, st, w, total_words, packed, sc, ze); break;
        default: {
            const long long groups = total_words / lpg;
            const int gblocks = static_cast<int>((groups + 7) / 8);
            quantize_warp_group_kernel<<<gblocks, 256, 0, st>>>(w, groups, lpg, packed, sc, ze, fmt);
        }
    }
    return launch_status();
}

size_t w4_workspace_bytes(int M, int N, int K, int transposed) {
    if (M <= 0 || N <= 0 || K <= 0 || K % 8 != 0) return 0;
    const int sms = device_info(current_device()).sms;
    if (M <= 4) return gemv_workspace(M, N, K, transposed, sms);
    return gemm_tc_workspace_bytes(M, N, K, transposed, sms);
}

w4_status w4a16_gemv(const void* A, int M, int N, int K, const uint32_t* packed,
                     const void* scales, const void* zeros, int mode, int group_size,
                     const void* bias, int transposed, void* Y, void* workspace,
                     size_t workspace_bytes, void* stream) {
    Meta meta;
    w4_status s = check_matmul(A, M, N, K, packed, scales, zeros, mode, group_size, bias, Y, &meta);
    if (s != W4_OK) return s;
    if (M > 4) return W4_ERR_INVALID_ARG;
    if (workspace && !aligned16(workspace)) return W4_ERR_ALIGNMENT;
    return run_gemv(A, M, N, K, packed, scales, zeros, meta, bias, transposed, Y, workspace,
                    workspace_bytes, static_cast<cudaStream_t>(stream));
}

w4_status w4a16_gemm(const void* A, int M, int N, int K, const uint32_t* packed,
                     const void* scales, const void* zeros, int mode, int group_size,
                     const void* bias, int transposed, void* Y, void* workspace,
                     size_t workspace_bytes, void* stream) {
    Meta meta;
    w4_status s = check_matmul(A, M, N, K, packed, scales, zeros, mode, group_size, bias, Y, &meta);
    if (s != W4_OK) return s;
    if (workspace && !aligned16(workspace)) return W4_ERR_ALIGNMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (M <= 4)
        return run_gemv(A, M, N, K, packed, scales, zeros, meta, bias, transposed, Y, workspace,
                        workspace_bytes, st);
    const int sms = device_info(current_device()).sms;
    if (workspace_bytes < gemm_tc_workspace_bytes(M, N, K, transposed, sms))
        return W4_ERR_WORKSPACE;
    TcProblem pr;
    pr.A = A;
    pr.M = M;
    pr.N = N;
    pr.K = K;
    pr.packed = packed;
    pr.S = scales;
    pr.Z = zeros;
    pr.g = meta.g;
    pr.G = meta.G;
    pr.sz_row = meta.sz_row;
    pr.fmt = meta.fmt;
    pr.bias = bias;
    pr.transposed = transposed;
    pr.Y = Y;
    pr.sms = sms;
    return run_gemm_tc(pr, workspace, workspace_bytes, st);
}

// Forward GEMV (M <= 4) that allocates nothing: its workspace goes to
// the library's built-in 8 MiB device scratch instead of a caller
// workspace.  See include/w4a16.h for who needs this and its limits.
w4_status w4a16_gemv_noalloc(const void* X, int M, int N, int K, const uint32_t* packed,
                             const void* scales, const void* zeros, int mode, int group_size,
                             const void* bias, void* Y, void* stream) {
    Meta meta;
    w4_status s = check_matmul(X, M, N, K, packed, scales, zeros, mode, group_size, bias, Y, &meta);
    if (s != W4_OK) return s;
    if (M > 4) return W4_ERR_INVALID_ARG;
    void* scratch = nullptr;
    s = noalloc_scratch(&scratch);
    if (s != W4_OK) return s;
    // the chosen plan's workspace is checked against the scratch size
    // before anything is launched (W4_ERR_WORKSPACE when it does not fit)
    return run_gemv_fwd(X, M, N, K, packed, scales, zeros, meta, bias, Y, scratch,
                        kNoAllocScratchBytes, static_cast<cudaStream_t>(stream));
}

const char* w4_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

w4_status w4_set_debug_checks(int on) {
    g_debug_checks.store(on ? 1 : 0, std::memory_order_relaxed);
    return W4_OK;
}

w4_status w4_debug_set_wait_limit(unsigned long long ns) {
    const unsigned long long v = ns ? ns : 2000000000ull;
    if (cudaMemcpyToSymbol(w4::g_wait_limit_ns, &v, sizeof v) != cudaSuccess) {
        g_last_cuda_error = cudaGetLastError();
        return W4_ERR_CUDA;
    }
    return W4_OK;
}

w4_status w4_debug_withhold_stage(int stage) {
    const int v = stage < 0 ? -1 : stage;
    if (cudaMemcpyToSymbol(w4::g_withhold_stage, &v, sizeof v) != cudaSuccess) {
        g_last_cuda_error = cudaGetLastError();
        return W4_ERR_CUDA;
    }
    return W4_OK;
}

uint64_t w4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

w4_status w4_device_error(int* code) {
    if (!code) return W4_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return W4_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, w4::g_error_word, sizeof v) != cudaSuccess) return W4_ERR_CUDA;
    if (cudaMemcpyToSymbol(w4::g_error_word, &zero, sizeof zero) != cudaSuccess) return W4_ERR_CUDA;
    *code = static_cast<int>(v);
    if (v == w4::kErrBadIndex) return W4_ERR_INVALID_ARG;
    return v ? W4_ERR_TIMEOUT : W4_OK;
}

// Rows up to this size are staged in shared memory by the column gather /
// scatter (two blocks per SM still fit).
constexpr size_t kRowStageBytes = 96u << 10;

w4_status w4_gather_columns(const void* A, int M, int src_cols, const int32_t* idx, int L, void* out,
                            void* stream) {
    if (M <= 0 || src_cols <= 0 || L <= 0 || !A || !idx || !out) return W4_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t row_bytes = (static_cast<size_t>(src_cols) * 2 + 15) & ~static_cast<size_t>(15);
    if (row_bytes <= kRowStageBytes) {
        if (ensure_smem(reinterpret_cast<const void*>(w4::gather_rows_kernel), row_bytes) != cudaSuccess)
            return W4_ERR_CUDA;
        const dim3 grid((L + w4::kGatherChunk - 1) / w4::kGatherChunk, std::min(M, 65535));
        launch_pdl(w4::gather_rows_kernel, grid, dim3(512), row_bytes, st, static_cast<const uint16_t*>(A), M,
                   src_cols, idx, L, static_cast<uint16_t*>(out));
        return launch_status();
    }
    const long long total = static_cast<long long>(M) * L;
    const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 148 * 16));
    w4::gather_columns_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint16_t*>(A), M, src_cols, idx, L,
                                                      static_cast<uint16_t*>(out));
    return launch_status();
}

w4_status w4_invert_permutation(const int32_t* perm, int n, int32_t* inv, void* stream) {
    if (n <= 0 || !perm || !inv) return W4_ERR_INVALID_ARG;
    const int blocks = std::min((n + 255) / 256, device_info(current_device()).sms * 4);
    launch_pdl(w4::invert_permutation_kernel, dim3(blocks), dim3(256), 0, static_cast<cudaStream_t>(stream), perm,
               n, inv);
    return launch_status();
}

w4_status w4_scatter_columns(const void* A, int M, int L, const int32_t* idx, int dst_cols, void* out,
                             void* stream) {
    if (M <= 0 || dst_cols <= 0 || L <= 0 || !A || !idx || !out) return W4_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t row_bytes = (static_cast<size_t>(dst_cols) * 2 + 15) & ~static_cast<size_t>(15);
    if (row_bytes <= kRowStageBytes) {
        if (ensure_smem(reinterpret_cast<const void*>(w4::scatter_rows_kernel), row_bytes) != cudaSuccess)
            return W4_ERR_CUDA;
        const int blocks = std::min(M, device_info(current_device()).sms * 4);
        launch_pdl(w4::scatter_rows_kernel, dim3(blocks), dim3(512), row_bytes, st, static_cast<const uint16_t*>(A),
                   M, L, idx, dst_cols, static_cast<uint16_t*>(out));
        return launch_status();
    }
    const long long total = static_cast<long long>(M) * L;
    const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 148 * 16));
    w4::scatter_columns_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint16_t*>(A), M, L, idx, dst_cols,
                                                       static_cast<uint16_t*>(out));
    return launch_status();
}

}  // extern "C"
