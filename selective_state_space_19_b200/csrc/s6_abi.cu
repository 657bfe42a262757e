// s6_abi.cu -- the C ABI declared in include/s6.h: argument checks, tensor-map
// set-up, kernel selection and launch.  Every arithmetic step of the path runs
// in the kernels of s6_scan.cuh, s6_conv.cuh and s6_step.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>

#include "s6.h"
#include "s6_common.cuh"
#include "s6_conv.cuh"
#include "s6_scan.cuh"
#include "s6_step.cuh"
#include "s6_bwd.cuh"
#include "s6_bwd_rev.cuh"
#include "s6_block.cuh"

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

// Every entry point restores the calling thread's current device before it
// returns: use_stream_device below may switch it to the stream's device.
struct DeviceRestore {
    int prev = -1;
    DeviceRestore() {
        if (cudaGetDevice(&prev) != cudaSuccess)
            prev = -1;
    }
    ~DeviceRestore() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev)
            cudaSetDevice(prev);
    }
    DeviceRestore(const DeviceRestore &) = delete;
    DeviceRestore &operator=(const DeviceRestore &) = delete;
};

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
// Library-owned scratch, one buffer per (device, use), allocated on first need
// and grown on demand (never while a stream is being captured); kept until
// process exit.  Uses: the scan's segment carries (a unit counter, flags,
// published states), and the backward's state checkpoints, its partial dB / dC
// rows and its reverse carries.
enum ScratchSlot { kScratchScan = 0, kScratchCkpt, kScratchPart, kScratchRev, kScratchBlock, kScratchSlots };
struct DeviceScratch {
    void *ptr = nullptr;
    size_t bytes = 0;
};
std::mutex g_scratch_mu;
DeviceScratch g_scratch[64][kScratchSlots];

int get_scratch(size_t bytes, cudaStream_t stream, void **out, int slot = kScratchScan) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return S6_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    DeviceScratch &sc = g_scratch[dev][slot];
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

// Fault injection for tests (s6_debug_carry_fault): off unless a test sets it.
constexpr unsigned int kCarryPolls = 1u << 22;  // ~0.3 s of polling at 64 ns sleeps
std::atomic<int> g_dbg_skip_publish{-1};
std::atomic<unsigned int> g_dbg_carry_polls{kCarryPolls};

// Whether a scan should use the associative split: too few (sequence, channel
// tile) chains to give a third of the CTA slots one each, and a sequence long
// enough to cut into segments of at least two chunks.
bool want_assoc(int64_t chains, int64_t L, int T, int64_t slots) {
    return chains > 0 && 3 * chains <= slots && L >= 4 * static_cast<int64_t>(T);
}

template <typename IO, int NS, int TPC, bool CONV, int MODE, int EXT>
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
    // the constant-decay form reads no step size: its dt map (never used) is built on x
    if (!make_map_3d(&tx, x, io, dims->batch, dims->seqlen, dims->d_inner, CPB, Sh::XR) ||
        !make_map_3d(&tdt, MODE == s6::kModeConst ? x : dt, io, dims->batch, dims->seqlen, dims->d_inner, CPB, T) ||
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
    constexpr bool INIT = EXT >= 1;
    auto kern = s6::s6_scan_kernel<IO, NS, TPC, T, STAGES, CONV, MODE, EXT>;
    const size_t smem = sizeof(Smem);
    // resident CTAs per SM for this instantiation, per device (the shared-memory
    // opt-in is a per-device attribute)
    static int occ_dev[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return S6_ERR_CUDA;
    if (!occ_dev[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess)
            return S6_ERR_CUDA;
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, s6::kScanBlock, smem) != cudaSuccess || nb < 1)
            return S6_ERR_CUDA;
        occ_dev[dev] = nb;
    }
    const int occ = occ_dev[dev];

    // ---- work split: chains of segments, pulled dynamically when there are
    // too few chains to balance the SMs statically
    const int64_t L = dims->seqlen;
    a.tiles = static_cast<int>((dims->d_inner + CPB - 1) / CPB);
    const int64_t chains = dims->batch * a.tiles;
    // Persistent CTAs, as many per SM as fit; no more of them than chains (or
    // units, for the associative split) can run at once.  With fewer chains
    // than CTA slots this still puts a second CTA on some SMs: measured on
    // Mamba-mini's 192 chains, 192 CTAs beat 148 (one per SM) by 2 %.
    const int64_t sms = device_sm_count();
    const bool assoc = INIT && want_assoc(chains, L, T, sms * occ);
    const int64_t per_sm = occ;
    const int64_t workers = sms * per_sm;
    int64_t nseg = 1, seg_len = round_up(static_cast<size_t>(L), T);
    if (assoc) {
        // Associative split: every chain's segments scan at once (segment 0 in
        // full, the others state-only from zero), then the later segments run
        // again from their folded start states.  Enough segments to give every
        // CTA slot a unit in the first phase, never shorter than 2 chunks.
        int64_t want = (workers + chains - 1) / chains;
        const int64_t max_seg = L / (2 * T);
        if (want > max_seg)
            want = max_seg;
        if (want < 2)
            want = 2;
        seg_len = round_up(static_cast<size_t>((L + want - 1) / want), T);
        nseg = (L + seg_len - 1) / seg_len;
    } else if (chains < 4 * workers && L > 4 * T) {
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
    a.assoc = assoc && nseg > 1;
    const int64_t units = a.assoc ? chains * (2 * nseg - 1) : chains * nseg;
    if (units > 0x7fffffffLL)
        return S6_ERR_UNSUPPORTED;
    a.nseg = static_cast<int>(nseg);
    a.seg_len = static_cast<int>(seg_len);
    a.units = static_cast<int>(units);
    a.dynamic = nseg > 1;
    a.carry_polls = g_dbg_carry_polls.load();
    a.skip_publish = g_dbg_skip_publish.load();
    unsigned grid = static_cast<unsigned>(chains);
    if (a.dynamic) {
        // serial: one flag per (chain, consumer warp) and one end state per
        // chain; associative: both per (chain, segment), plus the segments'
        // sums of Delta
        const size_t slots = static_cast<size_t>(chains) * (a.assoc ? nseg : 1);
        const size_t nflags = slots * s6::kConsumerWarps;
        const size_t hdr = round_up(4 + 4 * nflags, 256);
        const size_t carry = slots * CPB * NS * sizeof(float) + (a.assoc ? slots * CPB * sizeof(float) : 0);
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
        a.carry_sum = a.carry + slots * CPB * NS;
        if (cudaMemsetAsync(scr, 0, 4 + 4 * nflags, stream) != cudaSuccess)
            return S6_ERR_CUDA;
        const int64_t busy = a.assoc ? units : chains;  // units that can run at once
        grid = static_cast<unsigned>(busy < workers ? busy : workers);
    }
    kern<<<grid, s6::kScanBlock, smem, stream>>>(tx, tdt, tz, ty, tB, tC, a);
    return launch_status(cudaGetLastError());
}

template <typename IO, bool CONV, int MODE, int EXT>
int launch_scan_n(const s6_dims *dims, const void *x, const void *dt, const void *z, void *y, const ScanArgs &a,
                  cudaStream_t st, const FixedScratch *fixed = nullptr) {
    if constexpr (EXT >= 2) {  // checkpoints: N = 16 only (checked by the caller)
        return launch_scan_t<IO, 16, 2, CONV, MODE, EXT>(dims, x, dt, z, y, a, st, fixed);
    } else {
        if (dims->d_state <= 4)
            return launch_scan_t<IO, 4, 1, CONV, MODE, EXT>(dims, x, dt, z, y, a, st, fixed);
        if (dims->d_state <= 8)
            return launch_scan_t<IO, 8, 1, CONV, MODE, EXT>(dims, x, dt, z, y, a, st, fixed);
        return launch_scan_t<IO, 16, 2, CONV, MODE, EXT>(dims, x, dt, z, y, a, st, fixed);
    }
}

// Whether the problem has so few (sequence, channel tile) chains that the
// associative split pays (decided again with the kernel's occupancy at launch).
template <typename IO>
bool few_chains(const s6_dims *dims) {
    const int T = sizeof(IO) == 2 ? 64 : 32;
    const int64_t cpb = dims->d_state <= 8 ? 128 : 64;  // channels per CTA tile
    const int64_t chains = dims->batch * ((dims->d_inner + cpb - 1) / cpb);
    return want_assoc(chains, dims->seqlen, T, 2 * static_cast<int64_t>(device_sm_count()));
}

template <typename IO>
int launch_scan_io(const s6_dims *dims, bool conv, int mode, const void *x, const void *dt, const void *z, void *y,
                   const ScanArgs &a, cudaStream_t st, const FixedScratch *fixed = nullptr,
                   bool ckpt_outputs = false) {
    using s6::kModeConst;
    using s6::kModeSimplified;
    using s6::kModeZOH;
    if (mode == kModeConst)  // the constant-decay cell: no conv
        return (a.h_init || few_chains<IO>(dims)) ? launch_scan_n<IO, false, kModeConst, 1>(dims, x, dt, z, y, a, st, fixed)
                                                  : launch_scan_n<IO, false, kModeConst, 0>(dims, x, dt, z, y, a, st, fixed);
    const bool zoh = mode == kModeZOH;
    if (a.ckpt && ckpt_outputs) {  // a training forward: outputs and checkpoints
        if (conv)
            return zoh ? launch_scan_n<IO, true, kModeZOH, 3>(dims, x, dt, z, y, a, st, fixed)
                       : launch_scan_n<IO, true, kModeSimplified, 3>(dims, x, dt, z, y, a, st, fixed);
        return zoh ? launch_scan_n<IO, false, kModeZOH, 3>(dims, x, dt, z, y, a, st, fixed)
                   : launch_scan_n<IO, false, kModeSimplified, 3>(dims, x, dt, z, y, a, st, fixed);
    }
    if (a.ckpt) {  // the backward's checkpointing forward (no outputs)
        if (conv)
            return zoh ? launch_scan_n<IO, true, kModeZOH, 2>(dims, x, dt, z, y, a, st, fixed)
                       : launch_scan_n<IO, true, kModeSimplified, 2>(dims, x, dt, z, y, a, st, fixed);
        return zoh ? launch_scan_n<IO, false, kModeZOH, 2>(dims, x, dt, z, y, a, st, fixed)
                   : launch_scan_n<IO, false, kModeSimplified, 2>(dims, x, dt, z, y, a, st, fixed);
    }
    // the extended instantiation: a given start state, or the associative split
    if (a.h_init || a.conv_hist || few_chains<IO>(dims)) {
        if (conv)
            return zoh ? launch_scan_n<IO, true, kModeZOH, 1>(dims, x, dt, z, y, a, st, fixed)
                       : launch_scan_n<IO, true, kModeSimplified, 1>(dims, x, dt, z, y, a, st, fixed);
        return zoh ? launch_scan_n<IO, false, kModeZOH, 1>(dims, x, dt, z, y, a, st, fixed)
                   : launch_scan_n<IO, false, kModeSimplified, 1>(dims, x, dt, z, y, a, st, fixed);
    }
    if (conv)
        return zoh ? launch_scan_n<IO, true, kModeZOH, 0>(dims, x, dt, z, y, a, st, fixed)
                   : launch_scan_n<IO, true, kModeSimplified, 0>(dims, x, dt, z, y, a, st, fixed);
    return zoh ? launch_scan_n<IO, false, kModeZOH, 0>(dims, x, dt, z, y, a, st, fixed)
               : launch_scan_n<IO, false, kModeSimplified, 0>(dims, x, dt, z, y, a, st, fixed);
}

// mode: s6::kModeSimplified / kModeZOH (the zoh_mode argument of the scans) or
// kModeConst (s6_diag_recurrence_fwd's constant decay: A_log carries the log2
// of the decays, dt is not read).
int scan_common(const s6_dims *dims, bool conv, const void *x, const float *conv_w, const float *conv_b,
                const void *dt, const float *A_log, const void *B, const void *C, const float *D, const void *z,
                const float *dt_bias, int mode, void *y, float *h_final, s6_stream_t stream,
                const FixedScratch *fixed = nullptr, const float *h_init = nullptr,
                const void *conv_hist = nullptr, float *ckpt = nullptr, bool ckpt_outputs = false) {
    int st = check_dims(dims, true, conv);
    if (st != S6_OK)
        return st;
    if (mode != s6::kModeSimplified && mode != s6::kModeZOH && mode != s6::kModeConst)
        return S6_ERR_INVALID_ARG;
    const bool constd = mode == s6::kModeConst;
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
    if (!x || (!dt && !constd) || !A_log || !B || !C || !D || !y || (conv && !conv_w) || (constd && conv))
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
    a.ckpt = ckpt;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (use_stream_device(s) != S6_OK)
        return S6_ERR_CUDA;
    if (dims->io_dtype == S6_BF16)
        return launch_scan_io<__nv_bfloat16>(dims, conv, mode, x, dt, z, y, a, s, fixed, ckpt_outputs);
    return launch_scan_io<float>(dims, conv, mode, x, dt, z, y, a, s, fixed, ckpt_outputs);
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
    const int rc = get_scratch((ckf + hbf) * sizeof(float), st, &scr, kScratchCkpt);
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

// ------------------------------------------------- backward at N = 16 (pipelined)
// The reverse kernel over persistent CTAs: (segment, chain) units pulled
// last-segment-first when the chains alone would not balance the SMs.
template <typename IO, bool ZOH, bool CONV>
int launch_bwd_rev(const s6_dims *dims, s6::RevArgs r, const void *x, const void *dt, const void *z, const void *dy,
                   const void *B, const void *C, cudaStream_t st) {
    using Smem = s6::RevSmem<IO, CONV>;
    static_assert(offsetof(Smem, x) % 128 == 0 && offsetof(Smem, dt) % 128 == 0 && offsetof(Smem, z) % 128 == 0 &&
                      offsetof(Smem, dy) % 128 == 0 && offsetof(Smem, braw) % 128 == 0 &&
                      offsetof(Smem, craw) % 128 == 0,
                  "TMA buffers must be 128-byte aligned");
    static_assert(offsetof(Smem, hbuf) % 16 == 0 && offsetof(Smem, bc) % 16 == 0 && offsetof(Smem, full) % 8 == 0,
                  "vector and barrier fields must be aligned");
    auto kern = s6::s6_scan_bwd_rev_kernel<IO, ZOH, CONV>;
    const size_t smem = sizeof(Smem);
    static int occ_dev[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return S6_ERR_CUDA;
    if (!occ_dev[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess)
            return S6_ERR_CUDA;
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, s6::kScanBlock, smem) != cudaSuccess || nb < 1)
            return S6_ERR_CUDA;
        occ_dev[dev] = nb;
    }
    const int occ = occ_dev[dev];
    constexpr int KC = s6::kRevChunk;
    const int io = dims->io_dtype;
    CUtensorMap tx, tdt, tz, tdy, tB, tC;
    if (!make_map_3d(&tx, x, io, dims->batch, dims->seqlen, dims->d_inner, 64, Smem::XR) ||
        !make_map_3d(&tdt, dt, io, dims->batch, dims->seqlen, dims->d_inner, 64, KC) ||
        !make_map_3d(&tdy, dy, io, dims->batch, dims->seqlen, dims->d_inner, 64, KC) ||
        !make_map_3d(&tB, B, io, dims->batch, dims->seqlen, 16, 16, KC) ||
        !make_map_3d(&tC, C, io, dims->batch, dims->seqlen, 16, 16, KC))
        return S6_ERR_CUDA;
    if (z) {
        if (!make_map_3d(&tz, z, io, dims->batch, dims->seqlen, dims->d_inner, 64, KC))
            return S6_ERR_CUDA;
    } else {
        tz = tdt;  // never read
    }
    const int64_t L = dims->seqlen;
    const int64_t chains = dims->batch * r.tiles;
    const int64_t sms = device_sm_count();
    int64_t per_sm = occ;
    while (per_sm > 1 && per_sm * sms > chains)
        --per_sm;
    const int64_t workers = sms * per_sm;
    int64_t nseg = 1, seg_len = round_up(static_cast<size_t>(L), KC);
    if (chains < 4 * workers && L > 8 * KC) {
        // about 8 units per worker, segments of at least 8 sub-chunks
        const int64_t grid = chains < workers ? chains : workers;
        int64_t want = (8 * grid + chains - 1) / chains;
        const int64_t max_seg = L / (8 * KC);
        if (want > max_seg)
            want = max_seg;
        if (want > 1) {
            seg_len = round_up(static_cast<size_t>((L + want - 1) / want), KC);
            nseg = (L + seg_len - 1) / seg_len;
        }
    }
    if (chains * nseg > 0x7fffffffLL)
        return S6_ERR_UNSUPPORTED;
    r.nseg = static_cast<int>(nseg);
    r.seg_len = static_cast<int>(seg_len);
    r.units = static_cast<int>(chains * nseg);
    r.dynamic = nseg > 1;
    r.carry_polls = g_dbg_carry_polls.load();
    unsigned grid = static_cast<unsigned>(chains);
    if (r.dynamic) {
        const size_t nflags = static_cast<size_t>(chains) * s6::kConsumerWarps;
        const size_t hdr = round_up(4 + 4 * nflags, 256);
        const size_t carry = static_cast<size_t>(chains) * 64 * s6::kRevCarry * sizeof(float);
        void *scr = nullptr;
        const int rc = get_scratch(hdr + carry, st, &scr, kScratchRev);
        if (rc != S6_OK)
            return rc;
        r.counter = static_cast<unsigned int *>(scr);
        r.flags = r.counter + 1;
        r.carry = reinterpret_cast<float *>(static_cast<char *>(scr) + hdr);
        if (cudaMemsetAsync(scr, 0, 4 + 4 * nflags, st) != cudaSuccess)
            return S6_ERR_CUDA;
        grid = static_cast<unsigned>(chains < workers ? chains : workers);
    }
    kern<<<grid, s6::kScanBlock, smem, st>>>(tx, tdt, tz, tdy, tB, tC, r);
    return launch_status(cudaGetLastError());
}

// Whether the pipelined backward applies: N = 16 and rows that the tensor unit
// can move (16-byte aligned bases, d * sizeof(io) a multiple of 16).
bool bwd_rev_ok(const s6_dims *dims, const void *x, const void *dt, const void *z, const void *dy, const void *B,
                const void *C) {
    if (dims->d_state != 16 || (dims->d_inner * io_size(dims->io_dtype)) % 16 != 0)
        return false;
    const void *p[] = {x, dt, z, dy, B, C};
    for (const void *q : p)
        if (q && !aligned16(q))
            return false;
    return true;
}

// The pipelined backward: the forward kernel stores the state every
// kRevChunk tokens, the reverse kernel walks the chains back and writes
// per-tile dB / dC rows, and a reduction sums them over the tiles.
int bwd_rev(const s6_dims *dims, bool conv, const void *x, const float *conv_w, const float *conv_b, const void *dt,
            const float *A_log, const void *B, const void *C, const float *D, const void *z, const float *dt_bias,
            int zoh_mode, const float *h_init, const void *dy, float *dx, float *dconv_w, float *dconv_b, float *ddt,
            float *dz, float *dB, float *dC, float *dA_log, float *dD, float *ddt_bias, float *dh_init,
            cudaStream_t s, const float *ckpt_in = nullptr) {
    const int64_t Bt = dims->batch, L = dims->seqlen, d = dims->d_inner;
    const int64_t nck = (L + s6::kRevChunk - 1) / s6::kRevChunk;
    const int64_t tiles = (d + 63) / 64;
    void *ck = const_cast<float *>(ckpt_in), *pt = nullptr;
    int rc = ckpt_in ? S6_OK : get_scratch(sizeof(float) * Bt * nck * d * 16, s, &ck, kScratchCkpt);
    if (rc == S6_OK)
        rc = get_scratch(sizeof(float) * tiles * Bt * L * 32, s, &pt, kScratchPart);
    if (rc != S6_OK)
        return rc;
    // 1. the forward with checkpoints (no outputs), unless the caller's training
    // forward left them
    if (!ckpt_in) {
        const s6_dims fd = *dims;
        rc = scan_common(&fd, conv, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode,
                         const_cast<void *>(x), nullptr, reinterpret_cast<s6_stream_t>(s), nullptr, h_init, nullptr,
                         static_cast<float *>(ck));
        if (rc != S6_OK)
            return rc;
    }
    // 2. the reverse walk
    s6::RevArgs r;
    std::memset(&r, 0, sizeof(r));
    r.Bt = static_cast<int>(Bt);
    r.L = static_cast<int>(L);
    r.d = static_cast<int>(d);
    r.K = conv ? static_cast<int>(dims->conv_width) : 0;
    r.has_z = z != nullptr;
    r.tiles = static_cast<int>(tiles);
    r.nck = static_cast<int>(nck);
    r.A_log = A_log;
    r.D = D;
    r.dt_bias = dt_bias;
    r.conv_w = conv_w;
    r.conv_b = conv_b;
    r.ckpt = static_cast<const float *>(ck);
    r.du = dx;
    r.ddt = ddt;
    r.dz = dz;
    r.part = static_cast<float *>(pt);
    r.dA_log = dA_log;
    r.dD = dD;
    r.ddt_bias = ddt_bias;
    r.dconv_w = dconv_w;
    r.dconv_b = dconv_b;
    r.dh_init = dh_init;
    const bool zoh = zoh_mode == 1;
    if (dims->io_dtype == S6_BF16) {
        using T = __nv_bfloat16;
        rc = conv ? (zoh ? launch_bwd_rev<T, true, true>(dims, r, x, dt, z, dy, B, C, s)
                         : launch_bwd_rev<T, false, true>(dims, r, x, dt, z, dy, B, C, s))
                  : (zoh ? launch_bwd_rev<T, true, false>(dims, r, x, dt, z, dy, B, C, s)
                         : launch_bwd_rev<T, false, false>(dims, r, x, dt, z, dy, B, C, s));
    } else {
        rc = conv ? (zoh ? launch_bwd_rev<float, true, true>(dims, r, x, dt, z, dy, B, C, s)
                         : launch_bwd_rev<float, false, true>(dims, r, x, dt, z, dy, B, C, s))
                  : (zoh ? launch_bwd_rev<float, true, false>(dims, r, x, dt, z, dy, B, C, s)
                         : launch_bwd_rev<float, false, false>(dims, r, x, dt, z, dy, B, C, s));
    }
    if (rc != S6_OK)
        return rc;
    // 3. dB, dC over the tiles
    const long long rows = Bt * L;
    long long blocks = (rows * 32 + 255) / 256;
    const long long cap = static_cast<long long>(device_sm_count()) * 8;
    if (blocks > cap)
        blocks = cap;
    s6::s6_bwd_bc_reduce_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(static_cast<const float *>(pt),
                                                                             static_cast<int>(tiles), rows, dB, dC);
    return launch_status(cudaGetLastError());
}

// The backward entry points share their checks and set-up; `conv` selects the
// fused form (x, conv_w, conv_b in; dx, dconv_w, dconv_b out).
int bwd_common(const s6_dims *dims, bool conv, const void *x, const float *conv_w, const float *conv_b,
               const void *dt, const float *A_log, const void *B, const void *C, const float *D, const void *z,
               const float *dt_bias, int zoh_mode, const float *h_init, const void *dy, float *dx,
               float *dconv_w, float *dconv_b, float *ddt, float *dz, float *dB, float *dC, float *dA_log, float *dD,
               float *ddt_bias, float *dh_init, s6_stream_t stream, const float *ckpt_in = nullptr,
               bool from_ckpt = false) {
    int st = check_dims(dims, true, conv);
    if (st != S6_OK)
        return st;
    if (zoh_mode != 0 && zoh_mode != 1)
        return S6_ERR_INVALID_ARG;
    if (from_ckpt) {
        // the checkpoints of a training forward: the pipelined backward only
        if (!ckpt_in && dims->batch > 0 && dims->seqlen > 0)
            return S6_ERR_INVALID_ARG;
        if (dims->d_state != 16)
            return S6_ERR_UNSUPPORTED;
        if ((ckpt_in && !aligned16(ckpt_in)) || !bwd_rev_ok(dims, x, dt, z, dy, B, C))
            return S6_ERR_ALIGNMENT;
    }
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
    if (bwd_rev_ok(dims, x, dt, z, dy, B, C))
        return bwd_rev(dims, conv, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, h_init, dy, dx,
                       dconv_w, dconv_b, ddt, dz, dB, dC, dA_log, dD, ddt_bias, dh_init, s, ckpt_in);
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

// The training forwards: the scan with its outputs, also storing the state
// before every kCkptEvery-th token for a later s6_*_bwd_ckpt call.
int fwd_ckpt_common(const s6_dims *dims, bool conv, const void *x, const float *conv_w, const float *conv_b,
                    const void *dt, const float *A_log, const void *B, const void *C, const float *D, const void *z,
                    const float *dt_bias, int zoh_mode, const float *h_init, void *y, float *h_final, float *ckpt,
                    s6_stream_t stream) {
    int st = check_dims(dims, true, conv);
    if (st != S6_OK)
        return st;
    if (zoh_mode != 0 && zoh_mode != 1)
        return S6_ERR_INVALID_ARG;
    if (dims->d_state != 16)
        return S6_ERR_UNSUPPORTED;
    if (dims->batch > 0 && dims->seqlen > 0) {
        if (!ckpt)
            return S6_ERR_INVALID_ARG;
        if (!aligned16(ckpt))
            return S6_ERR_ALIGNMENT;
    }
    return scan_common(dims, conv, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, stream,
                       nullptr, h_init, nullptr, ckpt, true);
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
    DeviceRestore restore_device;
    if (zoh_mode != 0 && zoh_mode != 1)
        return S6_ERR_INVALID_ARG;
    return scan_common(dims, false, u, nullptr, nullptr, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final,
                       stream);
}

int s6_conv_scan_fwd(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b, const void *dt,
                     const float *A_log, const void *B, const void *C, const float *D, const void *z,
                     const float *dt_bias, int zoh_mode, void *y, float *h_final, s6_stream_t stream) {
    DeviceRestore restore_device;
    if (zoh_mode != 0 && zoh_mode != 1)
        return S6_ERR_INVALID_ARG;
    return scan_common(dims, true, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final,
                       stream);
}

int s6_conv_scan_fwd_noalloc(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b,
                             const void *dt, const float *A_log, const void *B, const void *C, const float *D,
                             const void *z, const float *dt_bias, int zoh_mode, void *y, float *h_final,
                             s6_stream_t stream) {
    DeviceRestore restore_device;
    if (zoh_mode != 0 && zoh_mode != 1)
        return S6_ERR_INVALID_ARG;
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
    DeviceRestore restore_device;
    if (zoh_mode != 0 && zoh_mode != 1)
        return S6_ERR_INVALID_ARG;
    return scan_common(dims, false, u, nullptr, nullptr, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final,
                       stream, nullptr, h_init, nullptr);
}

int s6_conv_scan_fwd_from_state(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b,
                                const void *dt, const float *A_log, const void *B, const void *C, const float *D,
                                const void *z, const float *dt_bias, int zoh_mode, const float *h_init,
                                const void *conv_hist, void *y, float *h_final, s6_stream_t stream) {
    DeviceRestore restore_device;
    if (zoh_mode != 0 && zoh_mode != 1)
        return S6_ERR_INVALID_ARG;
    return scan_common(dims, true, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, y, h_final, stream,
                       nullptr, h_init, conv_hist);
}

int s6_diag_recurrence_fwd(const s6_dims *dims, int decay_source, const void *u, const void *dt, const float *A_log,
                           const float *dt_bias, const float *log2_decay, const void *B, const void *C,
                           const float *D, const void *z, const float *h_init, void *y, float *h_final,
                           s6_stream_t stream) {
    DeviceRestore restore_device;
    if (decay_source == S6_DECAY_LIVE)
        return scan_common(dims, false, u, nullptr, nullptr, dt, A_log, B, C, D, z, dt_bias, s6::kModeSimplified, y,
                           h_final, stream, nullptr, h_init, nullptr);
    if (decay_source == S6_DECAY_CONST)
        return scan_common(dims, false, u, nullptr, nullptr, nullptr, log2_decay, B, C, D, z, nullptr,
                           s6::kModeConst, y, h_final, stream, nullptr, h_init, nullptr);
    return S6_ERR_INVALID_ARG;
}

int s6_scan_bwd(const s6_dims *dims, const void *u, const void *dt, const float *A_log, const void *B, const void *C,
                const float *D, const void *z, const float *dt_bias, int zoh_mode, const float *h_init, const void *dy,
                float *du, float *ddt, float *dz, float *dB, float *dC, float *dA_log, float *dD, float *ddt_bias,
                float *dh_init, s6_stream_t stream) {
    DeviceRestore restore_device;
    return bwd_common(dims, false, u, nullptr, nullptr, dt, A_log, B, C, D, z, dt_bias, zoh_mode, h_init, dy, du,
                      nullptr, nullptr, ddt, dz, dB, dC, dA_log, dD, ddt_bias, dh_init, stream);
}

int s6_conv_scan_bwd(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b, const void *dt,
                     const float *A_log, const void *B, const void *C, const float *D, const void *z,
                     const float *dt_bias, int zoh_mode, const float *h_init, const void *dy, float *dx,
                     float *dconv_w, float *dconv_b, float *ddt, float *dz, float *dB, float *dC, float *dA_log,
                     float *dD, float *ddt_bias, float *dh_init, s6_stream_t stream) {
    DeviceRestore restore_device;
    return bwd_common(dims, true, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, h_init, dy, dx,
                      dconv_w, dconv_b, ddt, dz, dB, dC, dA_log, dD, ddt_bias, dh_init, stream);
}

int s6_scan_fwd_ckpt(const s6_dims *dims, const void *u, const void *dt, const float *A_log, const void *B,
                     const void *C, const float *D, const void *z, const float *dt_bias, int zoh_mode,
                     const float *h_init, void *y, float *h_final, float *ckpt, s6_stream_t stream) {
    DeviceRestore restore_device;
    return fwd_ckpt_common(dims, false, u, nullptr, nullptr, dt, A_log, B, C, D, z, dt_bias, zoh_mode, h_init, y,
                           h_final, ckpt, stream);
}

int s6_conv_scan_fwd_ckpt(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b,
                          const void *dt, const float *A_log, const void *B, const void *C, const float *D,
                          const void *z, const float *dt_bias, int zoh_mode, const float *h_init, void *y,
                          float *h_final, float *ckpt, s6_stream_t stream) {
    DeviceRestore restore_device;
    return fwd_ckpt_common(dims, true, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, h_init, y,
                           h_final, ckpt, stream);
}

int s6_scan_bwd_ckpt(const s6_dims *dims, const void *u, const void *dt, const float *A_log, const void *B,
                     const void *C, const float *D, const void *z, const float *dt_bias, int zoh_mode,
                     const float *ckpt, const void *dy, float *du, float *ddt, float *dz, float *dB, float *dC,
                     float *dA_log, float *dD, float *ddt_bias, float *dh_init, s6_stream_t stream) {
    DeviceRestore restore_device;
    return bwd_common(dims, false, u, nullptr, nullptr, dt, A_log, B, C, D, z, dt_bias, zoh_mode, nullptr, dy, du,
                      nullptr, nullptr, ddt, dz, dB, dC, dA_log, dD, ddt_bias, dh_init, stream, ckpt, true);
}

int s6_conv_scan_bwd_ckpt(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b,
                          const void *dt, const float *A_log, const void *B, const void *C, const float *D,
                          const void *z, const float *dt_bias, int zoh_mode, const float *ckpt, const void *dy,
                          float *dx, float *dconv_w, float *dconv_b, float *ddt, float *dz, float *dB, float *dC,
                          float *dA_log, float *dD, float *ddt_bias, float *dh_init, s6_stream_t stream) {
    DeviceRestore restore_device;
    return bwd_common(dims, true, x, conv_w, conv_b, dt, A_log, B, C, D, z, dt_bias, zoh_mode, nullptr, dy, dx,
                      dconv_w, dconv_b, ddt, dz, dB, dC, dA_log, dD, ddt_bias, dh_init, stream, ckpt, true);
}

int causal_conv1d_silu_fwd(const s6_dims *dims, const void *x, const float *conv_w, const float *conv_b, void *out,
                           s6_stream_t stream) {
    DeviceRestore restore_device;
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
    DeviceRestore restore_device;
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

// Fault injection for tests: makes one unit of the next segmented scans skip
// publishing its carry, with a short poll limit, so that the successor's bounded
// wait runs out (S6_ERR_TIMEOUT through s6_device_status).  Host-side state only.
int s6_debug_carry_fault(int skip_publish_unit, unsigned int carry_polls) {
    g_dbg_skip_publish.store(skip_publish_unit < 0 ? -1 : skip_publish_unit);
    g_dbg_carry_polls.store(carry_polls == 0 ? kCarryPolls : carry_polls);
    return S6_OK;
}

int s6_block_step(const s6_block_dims *dims, const s6_block_weights *w, float *x, float *conv_state, float *h_ssm,
                  s6_stream_t stream) {
    DeviceRestore restore_device;
    if (!dims || !w)
        return S6_ERR_INVALID_ARG;
    const int64_t Bt = dims->batch, dm = dims->d_model, di = dims->d_inner, N = dims->d_state, R = dims->dt_rank,
                  K = dims->conv_width;
    if (Bt < 0 || dm < 1 || di < 1 || N < 1 || R < 1 || !(dims->eps >= 0.0f))
        return S6_ERR_INVALID_ARG;
    if (N > kMaxState || K < 2 || K > 4)
        return S6_ERR_UNSUPPORTED;
    if (Bt > (1 << 20) || dm > (1 << 20) || di > (1 << 24) || R > 1024)
        return S6_ERR_UNSUPPORTED;
    if (Bt == 0)
        return S6_OK;
    const void *req[] = {w->ln_w, w->ln_b, w->in_q, w->in_s, w->conv_w, w->xp_q, w->xp_s, w->dt_q, w->dt_s,
                         w->dt_bias, w->A_log, w->D, w->out_q, w->out_s, x, conv_state, h_ssm};
    for (const void *p : req)
        if (!p)
            return S6_ERR_INVALID_ARG;
    const void *f32p[] = {w->ln_w, w->ln_b, w->in_s, w->conv_w, w->conv_b, w->xp_s, w->dt_s, w->dt_bias, w->A_log,
                          w->D, w->out_s, x, conv_state, h_ssm};
    for (const void *p : f32p)
        if (p && !aligned_to(p, 4))
            return S6_ERR_ALIGNMENT;
    if (N == 16 && (!aligned16(w->A_log) || !aligned16(h_ssm)))
        return S6_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (use_stream_device(s) != S6_OK)
        return S6_ERR_CUDA;
    // intermediate rows: LayerNorm(x), xin | z, SiLU(conv(xin)), the x_proj rows
    // (dt | B | C), the gated readout -- each region a multiple of 4 floats
    const int64_t row = R + 2 * N;
    const size_t l_hn = round_up(static_cast<size_t>(dm), 4), l_xz = round_up(static_cast<size_t>(2 * di), 4),
                 l_xc = round_up(static_cast<size_t>(di), 4), l_dbc = round_up(static_cast<size_t>(row), 4);
    void *scr = nullptr;
    const size_t fl = static_cast<size_t>(Bt) * (l_hn + l_xz + l_xc + l_dbc + l_xc);
    int rc = get_scratch(fl * sizeof(float), s, &scr, kScratchBlock);
    if (rc != S6_OK)
        return rc;
    float *hn = static_cast<float *>(scr);
    float *xz = hn + static_cast<size_t>(Bt) * l_hn;
    float *xc = xz + static_cast<size_t>(Bt) * l_xz;
    float *dbc = xc + static_cast<size_t>(Bt) * l_xc;
    float *g = dbc + static_cast<size_t>(Bt) * l_dbc;
    const int64_t sms = device_sm_count();
    const unsigned mt = static_cast<unsigned>((Bt + s6::kGemmBM - 1) / s6::kGemmBM);
    // a product over the whole batch, Y = X W^T (add: Y += X W^T).  The
    // reduction is split across blocks (atomic adds; a Y that is overwritten is
    // zeroed first) until there are about three blocks per SM: the products are
    // short, and more blocks hide more of their load latency, but each split
    // adds every output once more (measured on the decode block, ms per token
    // step at 2 / 3 / 4 blocks per SM: 0.392 / 0.389 / 0.399).
    auto gemm = [&](const float *X, int ldx, int64_t n_out, int64_t k, const int8_t *wq, const float *ws, float *Y,
                    int ldy, bool add) -> int {
        const int64_t tiles = ((n_out + s6::kGemmBN - 1) / s6::kGemmBN) * mt;
        int64_t sp = (3 * sms + tiles - 1) / tiles;
        const int64_t max_sp = (k + s6::kGemmBK - 1) / s6::kGemmBK;
        if (sp > max_sp)
            sp = max_sp;
        if (sp < 1)
            sp = 1;
        if (sp > 1 && !add) {
            if (cudaMemset2DAsync(Y, sizeof(float) * ldy, 0, sizeof(float) * n_out, Bt, s) != cudaSuccess)
                return S6_ERR_CUDA;
            add = true;
        }
        const int64_t ks = round_up(static_cast<size_t>((k + sp - 1) / sp), s6::kGemmBK);
        s6::Q8GemmArgs ga;
        ga.M = static_cast<int>(Bt);
        ga.N = static_cast<int>(n_out);
        ga.K = static_cast<int>(k);
        ga.x = X;
        ga.ldx = ldx;
        ga.wq = wq;
        ga.ws = ws;
        ga.y = Y;
        ga.ldy = ldy;
        ga.accumulate = add ? 1 : 0;
        ga.k_split = static_cast<int>(ks);
        const dim3 grid(static_cast<unsigned>((n_out + s6::kGemmBN - 1) / s6::kGemmBN), mt,
                        static_cast<unsigned>((k + ks - 1) / ks));
        const bool vec = ldx % 4 == 0 && k % 8 == 0 && aligned16(X) && aligned_to(wq, 8);
        static int opted[64][2] = {};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
            return S6_ERR_CUDA;
        if (vec && k % 16 == 0 && aligned16(wq)) {
            // the tensor-core form (16-byte weight rows)
            static int opted_tc[64] = {};
            if (!opted_tc[dev]) {
                if (cudaFuncSetAttribute(s6::q8_tc_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(s6::kTcSmem)) != cudaSuccess)
                    return S6_ERR_CUDA;
                opted_tc[dev] = 1;
            }
            s6::q8_tc_gemm_kernel<<<grid, s6::kTcThreads, s6::kTcSmem, s>>>(ga);
            return cudaGetLastError() == cudaSuccess ? S6_OK : S6_ERR_CUDA;
        }
        if (!opted[dev][vec]) {
            const cudaError_t e =
                vec ? cudaFuncSetAttribute(s6::q8_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(s6::kGemmSmem))
                    : cudaFuncSetAttribute(s6::q8_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(s6::kGemmSmem));
            if (e != cudaSuccess)
                return S6_ERR_CUDA;
            opted[dev][vec] = 1;
        }
        if (vec)
            s6::q8_gemm_kernel<true><<<grid, s6::kGemmThreads, s6::kGemmSmem, s>>>(ga);
        else
            s6::q8_gemm_kernel<false><<<grid, s6::kGemmThreads, s6::kGemmSmem, s>>>(ga);
        return cudaGetLastError() == cudaSuccess ? S6_OK : S6_ERR_CUDA;
    };
    // 1. LayerNorm, then in_proj -> xin | z
    s6::block_layernorm_kernel<<<static_cast<unsigned>((Bt + 7) / 8), s6::kLnThreads, 0, s>>>(
        x, w->ln_w, w->ln_b, hn, static_cast<int>(Bt), static_cast<int>(dm), dims->eps);
    if (cudaGetLastError() != cudaSuccess)
        return S6_ERR_CUDA;
    rc = gemm(hn, static_cast<int>(dm), 2 * di, dm, w->in_q, w->in_s, xz, static_cast<int>(l_xz), false);
    if (rc != S6_OK)
        return rc;
    // 2. conv + SiLU (history shifted) and x_proj -> dt | B | C, a block per
    // sequence; 3. dt_proj + the recurrence + readout + gate -- at N = 16 in the
    // same block (xc and the x_proj row stay in shared memory)
    s6::BlockSsmArgs a3;
    a3.Bt = static_cast<int>(Bt);
    a3.di = static_cast<int>(di);
    a3.N = static_cast<int>(N);
    a3.R = static_cast<int>(R);
    a3.xz = xz;
    a3.xc = xc;
    a3.xz_ld = static_cast<int>(l_xz);
    a3.xc_ld = static_cast<int>(l_xc);
    a3.g_ld = static_cast<int>(l_xc);
    a3.dbc = dbc;
    a3.dbc_ld = static_cast<int>(l_dbc);
    a3.dt_q = w->dt_q;
    a3.dt_s = w->dt_s;
    a3.dt_bias = w->dt_bias;
    a3.A_log = w->A_log;
    a3.D = w->D;
    a3.h = h_ssm;
    a3.g = g;
    const bool fused = N == 16 && aligned16(h_ssm) && aligned16(w->A_log);
    {
        const size_t smem = sizeof(float) * (round_up(static_cast<size_t>(di), 4) + (fused ? row : 0));
        if (smem > 48 * 1024) {
            static int opted[64][2] = {};
            int dev = 0;
            if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
                return S6_ERR_CUDA;
            if (opted[dev][fused] < static_cast<int>(smem)) {
                if (smem > 227 * 1024 ||
                    cudaFuncSetAttribute(fused ? s6::block_conv_xproj_kernel<true> : s6::block_conv_xproj_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem)) != cudaSuccess)
                    return S6_ERR_UNSUPPORTED;
                opted[dev][fused] = static_cast<int>(smem);
            }
        }
        if (fused)
            s6::block_conv_xproj_kernel<true><<<static_cast<unsigned>(Bt), s6::kConvXThreads, smem, s>>>(
                xz, static_cast<int>(l_xz), w->conv_w, w->conv_b, conv_state, xc, static_cast<int>(l_xc), w->xp_q,
                w->xp_s, dbc, static_cast<int>(l_dbc), static_cast<int>(di), static_cast<int>(K), static_cast<int>(row),
                a3);
        else
            s6::block_conv_xproj_kernel<false><<<static_cast<unsigned>(Bt), s6::kConvXThreads, smem, s>>>(
                xz, static_cast<int>(l_xz), w->conv_w, w->conv_b, conv_state, xc, static_cast<int>(l_xc), w->xp_q,
                w->xp_s, dbc, static_cast<int>(l_dbc), static_cast<int>(di), static_cast<int>(K), static_cast<int>(row),
                a3);
        if (cudaGetLastError() != cudaSuccess)
            return S6_ERR_CUDA;
    }
    if (!fused) {
        s6::block_ssm_kernel<16><<<dim3(static_cast<unsigned>((di + s6::kSsmThreads - 1) / s6::kSsmThreads),
                                        static_cast<unsigned>(Bt)),
                                   s6::kSsmThreads, sizeof(float) * row, s>>>(a3);
        if (cudaGetLastError() != cudaSuccess)
            return S6_ERR_CUDA;
    }
    // 4. out_proj, added into the residual stream
    return gemm(g, static_cast<int>(l_xc), dm, di, w->out_q, w->out_s, x, static_cast<int>(dm), true);
}

// Read and clear the device-side error word after the stream's work so far
// (synchronises `stream`).  S6_ERR_TIMEOUT if a bounded wait gave up.
int s6_device_status(s6_stream_t stream) {
    DeviceRestore restore_device;
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
