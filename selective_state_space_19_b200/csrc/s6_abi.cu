// s6_abi.cu -- the C ABI declared in include/s6.h: argument checks, tensor-map
// set-up, kernel selection and launch.  Every arithmetic step of the path runs
// in the kernels of s6_scan.cuh, s6_conv.cuh and s6_step.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "s6.h"
#include "s6_common.cuh"
#include "s6_conv.cuh"
#include "s6_scan.cuh"
#include "s6_step.cuh"
#include "s6_bwd.cuh"

namespace {

using s6::ScanArgs;

constexpr int kMaxState = 16;

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D map over a [Bt, L, d] row-major tensor (dims innermost first: d, L, Bt)
// with a box of [1, rows, cols] elements.
bool make_map_3d(CUtensorMap *map, const void *base, int io, int64_t Bt, int64_t L, int64_t d, int box_cols,
                 int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const size_t es = io == S6_BF16 ? 2 : 4;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(Bt)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * es), static_cast<cuuint64_t>(L * d * es)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, io == S6_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void *p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

size_t io_size(int io) { return io == S6_BF16 ? 2 : 4; }

// ------------------------------------------------------------ validation
int check_dims(const s6_dims *dims, bool need_L, bool need_K) {
    if (!dims)
        return S6_ERR_INVALID_ARG;
    if (dims->batch < 0 || dims->seqlen < 0 || dims->d_inner < 1 || dims->d_state < 1)
        return S6_ERR_INVALID_ARG;
    if (dims->io_dtype != S6_F32 && dims->io_dtype != S6_BF16)
        return S6_ERR_UNSUPPORTED;
    if (dims->d_state > kMaxState)
        return S6_ERR_UNSUPPORTED;
    if (need_K && (dims->conv_width < 2 || dims->conv_width > 4))
        return S6_ERR_UNSUPPORTED;
    // 32-bit index arithmetic inside the kernels (per-sequence offsets stay 64-bit)
    if (dims->d_inner > (1 << 30) || dims->batch > (1 << 30) || (need_L && dims->seqlen > (1 << 30)))
        return S6_ERR_UNSUPPORTED;
    return S6_OK;
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? S6_OK : S6_ERR_CUDA; }

// Make the device that owns `stream` current for this library's runtime before
// any launch (the caller's framework may have selected it through another
// runtime instance in the same process).  The legacy and per-thread default
// streams keep the current device.
int use_stream_device(cudaStream_t stream) {
    if (stream == nullptr || stream == cudaStreamLegacy || stream == cudaStreamPerThread)
        return S6_OK;
    // a stream being captured into a graph: the capture already runs on the
    // current device, and device queries on it would invalidate the capture
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess)
        return S6_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone)
        return S6_OK;
    int dev = -1, cur = -1;
    if (cudaStreamGetDevice(stream, &dev) != cudaSuccess || cudaGetDevice(&cur) != cudaSuccess)
        return S6_ERR_CUDA;
    if (dev != cur && cudaSetDevice(dev) != cudaSuccess)
        return S6_ERR_CUDA;
    return S6_OK;
}

// ------------------------------------------------------------ scan dispatch
// Library-owned scratch for the dynamic scan: a unit counter, one flag per
// chain and one published end state per chain.  One buffer per device,
// allocated on first need and grown on demand (never while a stream is being
// captured); kept until process exit.
struct DeviceScratch {
    void *ptr = nullptr;
    size_t bytes = 0;
};
std::mutex g_scratch_mu;
DeviceScratch g_scratch[64];

int get_scratch(size_t bytes, cudaStream_t stream, void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return S6_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    DeviceScratch &sc = g_scratch[dev];
    if (sc.bytes < bytes) {
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        if (stream && cudaStreamIsCapturing(stream, &cap) != cudaSuccess)
            return S6_ERR_CUDA;
        if (cap != cudaStreamCaptureStatusNone)
            return S6_ERR_UNSUPPORTED;  // first (growing) call must come before capture
        if (sc.ptr && cudaFree(sc.ptr) != cudaSuccess)
            return S6_ERR_CUDA;
        sc.ptr = nullptr;
        sc.bytes = 0;
        const size_t want = bytes < (size_t(1) << 20) ? (size_t(1) << 20) : bytes;
        if (cudaMalloc(&sc.ptr, want) != cudaSuccess) {
            sc.ptr = nullptr;
            return S6_ERR_CUDA;
        }
        sc.bytes = want;
    }
    *out = sc.ptr;
    return S6_OK;
}

// A caller-independent scratch region of fixed size (see s6_conv_scan_fwd_noalloc).
struct FixedScratch {
    void *ptr;
    size_t bytes;
};

int device_sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

size_t round_up(size_t v, size_t m) { return (v + m - 1) / m * m; }

template <typename IO, int NS, int TPC, bool CONV, bool ZOH, bool INIT>
int launch_scan_t(const s6_dims *dims, const void *x, const void *dt, const void *z, void *y, ScanArgs a,
                  cudaStream_t stream, const FixedScratch *fixed = nullptr) {
    // Tokens per chunk: 64 (bf16) / 32 (f32).  A
    // chunk's first decays and first token quad are not overlapped with other
    // work, so long chunks amortise them; two stages of such chunks (about
    // 104 KB of shared memory) still leave room for two CTAs per SM.
    constexpr int T = sizeof(IO) == 2 ? 64 : 32;
    constexpr int STAGES = 2;
    using Sh = s6::ScanShape<NS, TPC, T, CONV>;
    using Smem = s6::ScanSmem<IO, NS, TPC, T, STAGES, CONV>;
    constexpr int CPB = Sh::CPB;
    // TMA destinations and sources must start on 128-byte boundaries
    static_assert(offsetof(Smem, x) % 128 == 0 && offsetof(Smem, dt) % 128 == 0 && offsetof(Smem, z) % 128 == 0 &&
                      offsetof(Smem, y) % 128 == 0 && offsetof(Smem, braw) % 128 == 0 &&
                      offsetof(Smem, craw) % 128 == 0 && sizeof(s6::Tile<IO, Sh::XR, CPB>) % 128 == 0,
                  "TMA buffers must be 128-byte aligned");
    static_assert(offsetof(Smem, bc) % 16 == 0 && offsetof(Smem, hinit) % 16 == 0 && offsetof(Smem, xch) % 16 == 0 &&
                      offsetof(Smem, meta) % 16 == 0 && offsetof(Smem, full) % 8 == 0,
                  "vector and barrier fields must be aligned");
    const int io = dims->io_dtype;
    const size_t es = io_size(io);
    CUtensorMap tx, tdt, tz, ty, tB, tC;
    if (!make_map_3d(&tx, x, io, dims->batch, dims->seqlen, dims->d_inner, CPB, Sh::XR) ||
        !make_map_3d(&tdt, dt, io, dims->batch, dims->seqlen, dims->d_inner, CPB, T) ||
        !make_map_3d(&ty, y, io, dims->batch, dims->seqlen, dims->d_inner, Sh::CPW, T))  // per-warp stores
        return S6_ERR_CUDA;
    if (z) {
        if (!make_map_3d(&tz, z, io, dims->batch, dims->seqlen, dims->d_inner, CPB, T))
            return S6_ERR_CUDA;
    } else {
        tz = tdt;  // never read when has_z == 0
    }
    // B/C rows by TMA when a row is a whole number of 16-byte units
    a.bc_tma = (dims->d_state * es) % 16 == 0 && aligned16(a.B) && aligned16(a.C);
    if (a.bc_tma) {
        if (!make_map_3d(&tB, a.B, io, dims->batch, dims->seqlen, dims->d_state, static_cast<int>(dims->d_state), T) ||
            !make_map_3d(&tC, a.C, io, dims->batch, dims->seqlen, dims->d_state, static_cast<int>(dims->d_state), T))
            return S6_ERR_CUDA;
    } else {
        tB = tC = tdt;  // never read
    }
    auto kern = s6::s6_scan_kernel<IO, NS, TPC, T, STAGES, CONV, ZOH, INIT>;
    const size_t smem = sizeof(Smem);
    static int occ = 0;  // resident CTAs per SM for this instantiation
    if (!occ) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess)
            return S6_ERR_CUDA;
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, s6::kScanBlock, smem) != cudaSuccess || nb < 1)
            return S6_ERR_CUDA;
        occ = nb;
    }

    // ---- work split: chains of segments, pulled dynamically when there are
    // too few chains to balance the SMs statically
    const int64_t L = dims->seqlen;
    a.tiles = static_cast<int>((dims->d_inner + CPB - 1) / CPB);
    const int64_t chains = dims->batch * a.tiles;
    // Every SM gets the same number of persistent CTAs, and no more CTAs run
    // than there are chains (a CTA beyond that would only wait).
    const int64_t sms = device_sm_count();
    int64_t per_sm = occ;
    while (per_sm > 1 && per_sm * sms > chains)
        --per_sm;
    const int64_t workers = sms * per_sm;
    int64_t nseg = 1, seg_len = round_up(static_cast<size_t>(L), T);
    if (chains < 4 * workers && L > 4 * T) {
        // about 16 units per worker: the last, partly filled wave of units is
        // short next to the whole run (a chain's segments run one after the
        // other, so at most `chains` units are ever in flight)
        const int64_t grid = chains < workers ? chains : workers;
        int64_t want = (16 * grid + chains - 1) / chains;
        const int64_t max_seg = L / (4 * T);
        if (want > max_seg)
            want = max_seg;
        if (want > 1) {
            seg_len = round_up(static_cast<size_t>((L + want - 1) / want), T);
            nseg = (L + seg_len - 1) / seg_len;
        }
    }
    if (chains * nseg > 0x7fffffffLL)
        return S6_ERR_UNSUPPORTED;
    a.nseg = static_cast<int>(nseg);
    a.seg_len = static_cast<int>(seg_len);
    a.units = static_cast<int>(chains * nseg);
    a.dynamic = nseg > 1;
    unsigned grid = static_cast<unsigned>(chains);
    if (a.dynamic) {
        const size_t nflags = static_cast<size_t>(chains) * s6::kConsumerWarps;
        const size_t hdr = round_up(4 + 4 * nflags, 256);
        const size_t carry = static_cast<size_t>(chains) * CPB * NS * sizeof(float);
        void *scr = nullptr;
        if (fixed) {
            if (hdr + carry > fixed->bytes)
                return S6_ERR_SCRATCH_LIMIT;
            scr = fixed->ptr;
        } else {
            const int st = get_scratch(hdr + carry, stream, &scr);
            if (st != S6_OK)
                return st;
        }
        a.counter = static_cast<unsigned int *>(scr);
        a.flags = a.counter + 1;
        a.carry = reinterpret_cast<float *>(static_cast<char *>(scr) + hdr);
        if (cudaMemsetAsync(scr, 0, 4 + 4 * nflags, stream) != cudaSuccess)
            return S6_ERR_CUDA;
        grid = static_cast<unsigned>(chains < workers ? chains : workers);
    }
    kern<<<grid, s6::kScanBlock, smem, stream>>>(tx, tdt, tz, ty, tB, tC, a);
    return launch_status(cudaGetLastError());
}

template <typename IO, bool CONV, bool ZOH, bool INIT>
int launch_scan_n(const s6_dims *dims, const void *x, const void *dt, const void *z, void *y, const ScanArgs &a,
                  cudaStream_t st, const FixedScratch *fixed = nullptr) {
    if (dims->d_state <= 4)
        return launch_scan_t<IO, 4, 1, CONV, ZOH, INIT>(dims, x, dt, z, y, a, st, fixed);
    if (dims->d_state <= 8)
        return launch_scan_t<IO, 8, 1, CONV, ZOH, INIT>(dims, x, dt, z, y, a, st, fixed);
    return launch_scan_t<IO, 16, 2, CONV, ZOH, INIT>(dims, x, dt, z, y, a, st, fixed);
}

template <typename IO>
int launch_scan_io(const s6_dims *dims, bool conv, bool zoh, const void *x, const void *dt, const void *z, void *y,
                   const ScanArgs &a, cudaStream_t st, const FixedScratch *fixed = nullptr) {
    if (a.h_init || a.conv_hist) {
        if (conv)
            return zoh ? launch_scan_n<IO, true, true, true>(dims, x, dt, z, y, a, st, fixed)
                       : launch_scan_n<IO, true, false, true>(dims, x, dt, z, y, a, st, fixed);
        return zoh ? launch_scan_n<IO, false, true, true>(dims, x, dt, z, y, a, st, fixed)
                   : launch_scan_n<IO, false, false, true>(dims, x, dt, z, y, a, st, fixed);
    }
    if (conv)
        return zoh ? launch_scan_n<IO, true, true, false>(dims, x, dt, z, y, a, st, fixed)
                   : launch_scan_n<IO, true, false, false>(dims, x, dt, z, y, a, st, fixed);
    return zoh ? launch_scan_n<IO, false, true, false>(dims, x, dt, z, y, a, st, fixed)
               : launch_scan_n<IO, false, false, false>(dims, x, dt, z, y, a, st, fixed);
}

int scan_common(const s6_dims *dims, bool conv, const void *x, const float *conv_w, const float *conv_b,
                const void *dt, const float *A_log, const void *B, const void *C, const float *D, const void *z,
                const float *dt_bias, int zoh_mode, void *y, float *h_final, s6_stream_t stream,
                const FixedScratch *fixed = nullptr, const float *h_init = nullptr,
                const void *conv_hist = nullptr) {
    int st = check_dims(dims, true, conv);
    if (st != S6_OK)
        return st;
    if (zoh_mode != 0 && zoh_mode != 1)
        return S6_ERR_INVALID_ARG;
    if ((h_init && !aligned_to(h_init, 4)) || (conv_hist && !aligned_to(conv_hist, io_size(dims->io_dtype))))
        return S6_ERR_ALIGNMENT;
    if (dims->batch == 0 || dims->seqlen == 0) {
        // nothing to scan; h_final of an empty sequence is the start state
        if (h_final && dims->batch > 0) {
            cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
            if (use_stream_device(s) != S6_OK)
                return S6_ERR_CUDA;
            const size_t bytes = sizeof(float) * dims->batch * dims->d_inner * dims->d_state;
            if (h_init)
                return launch_status(cudaMemcpyAsync(h_final, h_init, bytes, cudaMemcpyDeviceToDevice, s));
            return launch_status(cudaMemsetAsync(h_final, 0, bytes, s));
        }
        return S6_OK;
    }
    if (!x || !dt || !A_log || !B || !C || !D || !y || (conv && !conv_w))
        return S6_ERR_INVALID_ARG;
    const size_t es = io_size(dims->io_dtype);
    if ((dims->d_inner * es) % 16 != 0)
        return S6_ERR_ALIGNMENT;
    // rows moved by TMA need 16-byte aligned bases; the rest is read or
    // written element by element
    const void *tma_ptrs[] = {x, dt, y, z};
    for (const void *p : tma_ptrs)
        if (p && !aligned16(p))
            return S6_ERR_ALIGNMENT;
    const void *io_ptrs[] = {B, C};
    for (const void *p : io_ptrs)
        if (!aligned_to(p, es))
            return S6_ERR_ALIGNMENT;
    const void *f32_ptrs[] = {A_log, D, dt_bias, conv_w, conv_b, h_final};
    for (const void *p : f32_ptrs)
        if (p && !aligned_to(p, 4))
            return S6_ERR_ALIGNMENT;

    ScanArgs a;
    std::memset(&a, 0, sizeof(a));
    a.Bt = static_cast<int>(dims->batch);
    a.L = static_cast<int>(dims->seqlen);
    a.d = static_cast<int>(dims->d_inner);
    a.N = static_cast<int>(dims->d_state);
    a.has_z = z != nullptr;
    a.B = B;
    a.C = C;
    a.A_log = A_log;
    a.D = D;
    a.dt_bias = dt_bias;
    a.conv_w = conv ? conv_w : nullptr;
    a.conv_b = conv ? conv_b : nullptr;
    a.K = conv ? static_cast<int>(dims->conv_width) : 0;
    a.h_final = h_final;
    a.h_init = h_init;
    a.conv_hist = conv ? conv_hist : nullptr;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (use_stream_device(s) != S6_OK)
        return S6_ERR_CUDA;
    if (dims->io_dtype == S6_BF16)
        return launch_scan_io<__nv_bfloat16>(dims, conv, zoh_mode == 1, x, dt, z, y, a, s, fixed);
    return launch_scan_io<float>(dims, conv, zoh_mode == 1, x, dt, z, y, a, s, fixed);
}

// ------------------------------------------------------------ step dispatch
template <typename IO, int NS, bool ZOH>
int launch_step_t(const s6::StepArgs &a, cudaStream_t st) {
    const long long threads = static_cast<long long>(a.Bt) * a.d * (NS / 4);
    const long long blocks = (threads + s6::kStepThreads - 1) / s6::kStepThreads;
    if (blocks > 0x7fffffffLL)
        return S6_ERR_UNSUPPORTED;
    s6::s6_step_kernel<IO, NS, ZOH><<<static_cast<unsigned>(blocks), s6::kStepThreads, 0, st>>>(a);
    return launch_status(cudaGetLastError());
}

// N in {4, 8, 16}: the pipelined kernel over persistent CTAs, each walking one
// contiguous range of (channel tile, sequence) tiles.  BIO: the per-token rows
// also move by bulk copies (all their runs 16-byte aligned).
template <typename IO, int NS, bool ZOH, bool BIO>
int launch_step_bulk(const s6::StepArgs &a, cudaStream_t st) {
    constexpr int CT = s6::kStepThreads;  // channels per tile
    static int occ[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return S6_ERR_CUDA;
    if (!occ[dev]) {
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, s6::s6_step_bulk_kernel<IO, NS, ZOH, BIO>,
                                                          s6::kStepThreads, 0) != cudaSuccess ||
            nb < 1)
            return S6_ERR_CUDA;
        occ[dev] = nb;
    }
    const long long ctiles = (a.d + CT - 1) / CT;
    const long long ntiles = ctiles * a.Bt;
    if (ntiles == 0)
        return S6_OK;
    const long long max_grid = static_cast<long long>(device_sm_count()) * occ[dev];
    const long long per = (ntiles + max_grid - 1) / max_grid;  // tiles per CTA, balanced
    const long long grid = (ntiles + per - 1) / per;
    if (grid > 0x7fffffffLL || per > 0x7fffffffLL)
        return S6_ERR_UNSUPPORTED;
    s6::s6_step_bulk_kernel<IO, NS, ZOH, BIO><<<static_cast<unsigned>(grid), s6::kStepThreads, 0, st>>>(
        a, static_cast<int>(ctiles), static_cast<int>(per));
    return launch_status(cudaGetLastError());
}

// Whether every per-token run of a tile starts and ends on 16 bytes: the rows
// of u, Delta, z, y and the conv history are [batch, d_inner(, K-1)] with
// element size es, so d_inner * es must be a multiple of 16 and the base
// pointers 16-byte aligned.
bool step_rows_bulk(const s6::StepArgs &a, size_t es) {
    if ((static_cast<size_t>(a.d) * es) % 16 != 0)
        return false;
    const void *p[] = {a.u, a.dt, a.z, a.conv_state, a.y};
    for (const void *q : p)
        if (q && !aligned_to(q, 16))
            return false;
    return true;
}

template <typename IO, int NS, bool ZOH>
int launch_step_bulk_io(const s6::StepArgs &a, cudaStream_t st) {
    return step_rows_bulk(a, sizeof(IO)) ? launch_step_bulk<IO, NS, ZOH, true>(a, st)
                                         : launch_step_bulk<IO, NS, ZOH, false>(a, st);
}

template <typename IO, bool ZOH>
int launch_step_n(const s6::StepArgs &a, cudaStream_t st) {
    if (a.N == 4)
        return launch_step_bulk_io<IO, 4, ZOH>(a, st);
    if (a.N == 8)
        return launch_step_bulk_io<IO, 8, ZOH>(a, st);
    if (a.N == 16)
        return launch_step_bulk_io<IO, 16, ZOH>(a, st);
    if (a.N < 4)
        return launch_step_t<IO, 4, ZOH>(a, st);
    if (a.N < 8)
        return launch_step_t<IO, 8, ZOH>(a, st);
    return launch_step_t<IO, 16, ZOH>(a, st);
}

// ------------------------------------------------ scratch that is never allocated
// The carry scratch of s6_conv_scan_fwd_noalloc: one fixed array in the
// library's device image, present on every GPU that loads the library until
// the process exits.  Host code must not pass this name to a kernel (on the host
// it only stands for the symbol); its device address is looked up once per
// device with cudaGetSymbolAddress while that device is current.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_s6_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_addr[64] = {nullptr};

// Device address of the fixed scratch on the device that owns `stream`.
int noalloc_scratch(cudaStream_t stream, FixedScratch *out) {
    if (use_stream_device(stream) != S6_OK)
        return S6_ERR_CUDA;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return S6_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_s6_noalloc_scratch) != cudaSuccess || p == nullptr)
            return S6_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    out->ptr = g_noalloc_addr[dev];
    out->bytes = kNoAllocScratchBytes;
    return S6_OK;
}

}  // namespace

// ======================================================================= ABI
// Persistent CTAs (as many as fit on the SMs) over balanced contiguous ranges
// of (channel tile, sequence, token tile) tiles.
template <typename IO>
int launch_conv(const s6_dims *dims, const void *x, s6::ConvArgs a, cudaStream_t st) {
    using Sh = s6::ConvShape<IO>;
    auto kern = s6::s6_conv_silu_kernel<IO>;
    constexpr size_t smem = sizeof(s6::ConvSmem<IO>);
    static int occ[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return S6_ERR_CUDA;
    if (!occ[dev]) {
        int nb = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
                cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, 32 * s6::kConvWarps, smem) != cudaSuccess ||
            nb < 1)
            return S6_ERR_CUDA;
        occ[dev] = nb;
    }
    CUtensorMap tx;
    if (!make_map_3d(&tx, x, dims->io_dtype, dims->batch, dims->seqlen, dims->d_inner, Sh::CC, s6::kConvT + 3))
        return S6_ERR_CUDA;
    const long long ctiles = (dims->d_inner + Sh::CC - 1) / Sh::CC;
    const long long ttiles = (dims->seqlen + s6::kConvT - 1) / s6::kConvT;
    const long long ntiles = ctiles * dims->batch * ttiles;
    const long long max_grid = static_cast<long long>(device_sm_count()) * occ[dev];
    const long long per = (ntiles + max_grid - 1) / max_grid;  // tiles per CTA, balanced
    const long long grid = (ntiles + per - 1) / per;
    if (grid > 0x7fffffffLL || per > 0x7fffffffLL || ttiles > 0x7fffffffLL)
        return S6_ERR_UNSUPPORTED;
    a.ctiles = static_cast<int>(ctiles);
    a.ttiles = static_cast<int>(ttiles);
    a.per_cta = static_cast<int>(per);
    kern<<<static_cast<unsigned>(grid), 32 * s6::kConvWarps, smem, st>>>(tx, a);
    return launch_status(cudaGetLastError());
}

// ------------------------------------------------------------ backward dispatch
// Checkpoints and chunk states live in the library-owned scratch buffer.
template <typename IO, int NS, bool ZOH, bool CONV>
int launch_bwd_t(s6::BwdArgs a, cudaStream_t st) {
    const long long G = static_cast<long long>(a.Bt) * a.d;
    const size_t ckf = static_cast<size_t>(a.nck) * NS * G;
    const size_t hbf = static_cast<size_t>(s6::kBwdChunk) * NS * G;
    void *scr = nullptr;
    const int rc = get_scratch((ckf + hbf) * sizeof(float), st, &scr);
    if (rc != S6_OK)
        return rc;
    a.ck = static_cast<float *>(scr);
    a.hb = a.ck + ckf;
    const long long grid = (G * s6::kBwdTPC + s6::kBwdThreads - 1) / s6::kBwdThreads;
    if (grid > 0x7fffffffLL)
        return S6_ERR_UNSUPPORTED;
    s6::s6_scan_bwd_kernel<IO, NS, ZOH, CONV><<<static_cast<unsigned>(grid), s6::kBwdThreads, 0, st>>>(a);
    return launch_status(cudaGetLastError());
}

template <typename IO, bool ZOH, bool CONV>
int launch_bwd_n(const s6::BwdArgs &a, cudaStream_t st) {
    if (a.N <= 4)
        return launch_bwd_t<IO, 4, ZOH, CONV>(a, st);
    if (a.N <= 8)
        return launch_bwd_t<IO, 8, ZOH, CONV>(a, st);
    return launch_bwd_t<IO, 16, ZOH, CONV>(a, st);
}

template <typename IO>
int launch_bwd_io(const s6::BwdArgs &a, bool zoh, bool conv, cudaStream_t st) {
    if (conv)
        return zoh ? launch_bwd_n<IO, true, true>(a, st) : launch_bwd_n<IO, false, true>(a, st);
    return zoh ? launch_bwd_n<IO, true, false>(a, st) : launch_bwd_n<IO, false, false>(a, st);
}

// The backward entry points share their checks and set-up; `conv` selects the
// fused form (x, conv_w, conv_b in; dx, dconv_w, dconv_b out).
int bwd_common(const s6_dims *dims, bool conv, const void *x, const float *conv_w, const float *conv_b,
               const void *dt, const float *A_log, const void *B, const void *C, const float *D, const void *z,
               const float *dt_bias, int zoh_mode, const float *h_init, const void *dy, float *dx,
               float *dconv_w, float *dconv_b, float *ddt, float *dz, float *dB, float *dC, float *dA_log, float *dD,
               float *ddt_bias, float *dh_init, s6_stream_t stream) {
    int st = check_dims(dims, true, conv);
    if (st != S6_OK)
        return st;
    if (zoh_mode != 0 && zoh_mode != 1)
        return S6_ERR_INVALID_ARG;
    if (dims->batch == 0)
        return S6_OK;
    if (!x || !dt || !A_log || !B || !C || !D || !dy || !dx || !ddt || !dB || !dC || !dA_log || !dD || (z && !dz) ||
        (conv && (!conv_w || !dconv_w)))
        return S6_ERR_INVALID_ARG;
    const size_t es = io_size(dims->io_dtype);
    const void *io_ptrs[] = {x, dt, B, C, z, dy};
    for (const void *p : io_ptrs)
        if (p && !aligned_to(p, es))
            return S6_ERR_ALIGNMENT;
    const void *f32_ptrs[] = {A_log, D, dt_bias, h_init, conv_w, conv_b, dx, ddt, dz, dB, dC, dA_log, dD,
                              ddt_bias, dh_init, dconv_w, dconv_b};
    for (const void *p : f32_ptrs)
        if (p && !aligned_to(p, 4))
            return S6_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (use_stream_device(s) != S6_OK)
        return S6_ERR_CUDA;
    // the summed gradients start from zero
    const int64_t Bt = dims->batch, L = dims->seqlen, d = dims->d_inner, N = dims->d_state;
    const int64_t K = conv ? dims->conv_width : 0;
    if (cudaMemsetAsync(dB, 0, sizeof(float) * Bt * L * N, s) != cudaSuccess ||
        cudaMemsetAsync(dC, 0, sizeof(float) * Bt * L * N, s) != cudaSuccess ||
        cudaMemsetAsync(dA_log, 0, sizeof(float) * d * N, s) != cudaSuccess ||
        cudaMemsetAsync(dD, 0, sizeof(float) * d, s) != cudaSuccess ||
        (ddt_bias && cudaMemsetAsync(ddt_bias, 0, sizeof(float) * d, s) != cudaSuccess) ||
        (conv && cudaMemsetAsync(dconv_w, 0, sizeof(float) * d * K, s) != cudaSuccess) ||
        (conv && dconv_b && cudaMemsetAsync(dconv_b, 0, sizeof(float) * d, s) != cudaSuccess))
        return S6_ERR_CUDA;
    if (L == 0) {
        // an empty sequence contributes nothing; the start state gets no gradient
        if (dh_init && cudaMemsetAsync(dh_init, 0, sizeof(float) * Bt * d * N, s) != cudaSuccess)
            return S6_ERR_CUDA;
        return S6_OK;
    }
    s6::BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.Bt = static_cast<int>(Bt);
    a.L = static_cast<int>(L);
    a.d = static_cast<int>(d);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.has_z = z != nullptr;
    a.nck = static_cast<int>((L + s6::kBwdChunk - 1) / s6::kBwdChunk);
    a.u = x;
    a.dt = dt;
    a.B = B;
    a.C = C;
    a.z = z;
    a.dy = dy;
    a.A_log = A_log;
    a.D = D;
    a.dt_bias = dt_bias;
    a.h_init = h_init;
    a.conv_w = conv_w;
    a.conv_b = conv_b;
    a.du = dx;
    a.ddt = ddt;
    a.dz = dz;
    a.dB = dB;
    a.dC = dC;
    a.dA_log = dA_log;
    a.dD = dD;
    a.ddt_bias = ddt_bias;
    a.dh_init = dh_init;
    a.dconv_w = dconv_w;
    a.dconv_b = dconv_b;
    if (dims->io_dtype == S6_BF16)
        return launch_bwd_io<__nv_bfloat16>(a, zoh_mode == 1, conv, s);
    return launch_bwd_io<float>(a, zoh_mode == 1, conv, s);
}

extern "C" {

int s6_version(void) { return (1 << 16) | 0; }

const char *s6_status_string(int status) {
    switch (status) {
        case S6_OK: return "S6_OK";
        case S6_ERR_INVALID_ARG: return "S6_ERR_INVALID_ARG: null pointer or invalid size";
        case S6_ERR_UNSUPPORTED: return "S6_ERR_UNSUPPORTED: size, width or dtype outside the supported range";
        case S6_ERR_ALIGNMENT: return "S6_ERR_ALIGNMENT: pointer or row not 16-byte aligned";
        case S6_ERR_CUDA: return "S6_ERR_CUDA: a CUDA call or kernel launch failed";
        case S6_ERR_TIMEOUT: return "S6_ERR_TIMEOUT: a bounded device-side wait gave up";
        case S6_ERR_SCRATCH_LIMIT:
            return "S6_ERR_SCRATCH_LIMIT: the problem needs more carry scratch than the fixed 4 MiB array holds";
        default: return "S6: unknown status";
    }
}

int s6_scan_fwd(const s6_dims *dims, const void *u, const void *dt, const float *A_log, const void *B, const void *C,
                const float *D, const void *z, const float *dt_bias, int zoh_mode, void *y, float *h_final,
                s6_stream_t stream) {
    return scan_common(dims, false, u, nullptr, nullptr, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final,
                       stream);
}

int s6_conv_scan_fwd(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b, const void *dt,
                     const float *A_log, const void *B, const void *C, const float *D, const void *z,
                     const float *dt_bias, int zoh_mode, void *y, float *h_final, s6_stream_t stream) {
    return scan_common(dims, true, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final,
                       stream);
}

int s6_conv_scan_fwd_noalloc(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b,
                             const void *dt, const float *A_log, const void *B, const void *C, const float *D,
                             const void *z, const float *dt_bias, int zoh_mode, void *y, float *h_final,
                             s6_stream_t stream) {
    FixedScratch fx;
    const int st = noalloc_scratch(reinterpret_cast<cudaStream_t>(stream), &fx);
    if (st != S6_OK)
        return st;
    return scan_common(dims, true, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, stream,
                       &fx);
}

int s6_scan_fwd_from_state(const s6_dims *dims, const void *u, const void *dt, const float *A_log, const void *B,
                           const void *C, const float *D, const void *z, const float *dt_bias, int zoh_mode,
                           const float *h_init, void *y, float *h_final, s6_stream_t stream) {
    return scan_common(dims, false, u, nullptr, nullptr, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final,
                       stream, nullptr, h_init, nullptr);
}

int s6_conv_scan_fwd_from_state(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b,
                                const void *dt, const float *A_log, const void *B, const void *C, const float *D,
                                const void *z, const float *dt_bias, int zoh_mode, const float *h_init,
                                const void *conv_hist, void *y, float *h_final, s6_stream_t stream) {
    return scan_common(dims, true, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, stream,
                       nullptr, h_init, conv_hist);
}

int s6_scan_bwd(const s6_dims *dims, const void *u, const void *dt, const float *A_log, const void *B, const void *C,
                const float *D, const void *z, const float *dt_bias, int zoh_mode, const float *h_init, const void *dy,
                float *du, float *ddt, float *dz, float *dB, float *dC, float *dA_log, float *dD, float *ddt_bias,
                float *dh_init, s6_stream_t stream) {
    return bwd_common(dims, false, u, nullptr, nullptr, dt, A_log, B, C, D, z, dt_bias, zoh_mode, h_init, dy, du,
                      nullptr, nullptr, ddt, dz, dB, dC, dA_log, dD, ddt_bias, dh_init, stream);
}

int s6_conv_scan_bwd(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b, const void *dt,
                     const float *A_log, const void *B, const void *C, const float *D, const void *z,
                     const float *dt_bias, int zoh_mode, const float *h_init, const void *dy, float *dx,
                     float *dconv_w, float *dconv_b, float *ddt, float *dz, float *dB, float *dC, float *dA_log,
                     float *dD, float *ddt_bias, float *dh_init, s6_stream_t stream) {
    return bwd_common(dims, true, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, h_init, dy, dx,
                      dconv_w, dconv_b, ddt, dz, dB, dC, dA_log, dD, ddt_bias, dh_init, stream);
}

int causal_conv1d_silu_fwd(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b, void *out,
                           s6_stream_t stream) {
    int st = check_dims(dims, true, true);
    if (st != S6_OK)
        return st;
    if (dims->batch == 0 || dims->seqlen == 0)
        return S6_OK;
    if (!x || !conv_w || !out)
        return S6_ERR_INVALID_ARG;
    if ((dims->d_inner * io_size(dims->io_dtype)) % 16 != 0)
        return S6_ERR_ALIGNMENT;
    if (!aligned16(x) || !aligned16(out) || !aligned_to(conv_w, 4) || (conv_b && !aligned_to(conv_b, 4)))
        return S6_ERR_ALIGNMENT;
    s6::ConvArgs a;
    a.Bt = static_cast<int>(dims->batch);
    a.L = static_cast<int>(dims->seqlen);
    a.d = static_cast<int>(dims->d_inner);
    a.K = static_cast<int>(dims->conv_width);
    a.x = x;
    a.conv_w = conv_w;
    a.conv_b = conv_b;
    a.out = out;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (use_stream_device(s) != S6_OK)
        return S6_ERR_CUDA;
    return dims->io_dtype == S6_BF16 ? launch_conv<__nv_bfloat16>(dims, x, a, s) : launch_conv<float>(dims, x, a, s);
}

int s6_step(const s6_dims *dims, const float *A_log, const float *D, const float *dt_bias, const float *conv_w,
            const float *conv_b, int zoh_mode, const void *u_t, const void *dt_t, const void *B_t, const void *C_t,
            const void *z_t, float *h_ssm, void *conv_state, void *y_t, s6_stream_t stream) {
    int st = check_dims(dims, false, true);
    if (st != S6_OK)
        return st;
    if (zoh_mode != 0 && zoh_mode != 1)
        return S6_ERR_INVALID_ARG;
    if (dims->batch == 0)
        return S6_OK;
    if (!A_log || !D || !conv_w || !u_t || !dt_t || !B_t || !C_t || !h_ssm || !conv_state || !y_t)
        return S6_ERR_INVALID_ARG;
    // h_ssm and A_log rows are moved 16 bytes at a time when N is 4, 8 or 16;
    // everything else element by element
    const size_t es = io_size(dims->io_dtype);
    const bool vec = dims->d_state == 4 || dims->d_state == 8 || dims->d_state == 16;
    if (!aligned_to(h_ssm, vec ? 16 : 4) || !aligned_to(A_log, vec ? 16 : 4))
        return S6_ERR_ALIGNMENT;
    const void *f32_ptrs[] = {D, dt_bias, conv_w, conv_b};
    for (const void *p : f32_ptrs)
        if (p && !aligned_to(p, 4))
            return S6_ERR_ALIGNMENT;
    const void *io_ptrs[] = {u_t, dt_t, B_t, C_t, z_t, conv_state, y_t};
    for (const void *p : io_ptrs)
        if (p && !aligned_to(p, es))
            return S6_ERR_ALIGNMENT;
    s6::StepArgs a;
    a.Bt = static_cast<int>(dims->batch);
    a.d = static_cast<int>(dims->d_inner);
    a.N = static_cast<int>(dims->d_state);
    a.K = static_cast<int>(dims->conv_width);
    a.zoh = zoh_mode;
    a.has_z = z_t != nullptr;
    a.A_log = A_log;
    a.D = D;
    a.dt_bias = dt_bias;
    a.conv_w = conv_w;
    a.conv_b = conv_b;
    a.u = u_t;
    a.dt = dt_t;
    a.B = B_t;
    a.C = C_t;
    a.z = z_t;
    a.h = h_ssm;
    a.conv_state = conv_state;
    a.y = y_t;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (use_stream_device(s) != S6_OK)
        return S6_ERR_CUDA;
    if (dims->io_dtype == S6_BF16)
        return zoh_mode ? launch_step_n<__nv_bfloat16, true>(a, s) : launch_step_n<__nv_bfloat16, false>(a, s);
    return zoh_mode ? launch_step_n<float, true>(a, s) : launch_step_n<float, false>(a, s);
}

// Read and clear the device-side error word after the stream's work so far
// (synchronises `stream`).  S6_ERR_TIMEOUT if a bounded wait gave up.
int s6_device_status(s6_stream_t stream) {
    unsigned int v = 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (use_stream_device(s) != S6_OK)
        return S6_ERR_CUDA;
    if (cudaMemcpyFromSymbolAsync(&v, s6::g_s6_device_error, sizeof(v), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return S6_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return S6_ERR_CUDA;
    if (v) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbolAsync(s6::g_s6_device_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) !=
            cudaSuccess)
            return S6_ERR_CUDA;
        cudaStreamSynchronize(s);
        return S6_ERR_TIMEOUT;
    }
    return S6_OK;
}

}  // extern "C"
