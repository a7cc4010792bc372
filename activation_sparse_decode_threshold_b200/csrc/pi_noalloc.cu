// pi_noalloc.cu -- pi_predict_noalloc: the low-rank predictor on caller-owned
// weights with no device allocation anywhere on its path.
//
// Who needs it: code that must not call cudaMalloc at the point where it
// predicts -- for example a serving loop whose device memory budget is fully
// committed to weights and KV caches at start-up, an allocator-owning host
// runtime that forbids other libraries from allocating behind its back, or a
// caller that has no handle at all (pi_ffn_create allocates the handle's
// scratch and tables).  It runs the same predictor arithmetic as pi_predict
// (the decode kernel in predictor mode, rows of t = V x split over the CTAs)
// with every byte of scratch in one file-scope __device__ array, and takes
// the weights as they are (row-major, original neuron order, no neuron table).
#include <cmath>
#include <cstdio>
#include <mutex>

#include "../../include/pi_ffn.h"
#include "pi_internal.h"

namespace {

// Scratch layout (bytes), for up to kMaxStrips strips:
//   lists    kMaxStrips * kMaxStrip ints  per-strip active lists
//   counts   kMaxStrips ints              per-strip active counts
//   bar      kBarWords unsigned           grid barrier counter, tagged slots of t (zeroed per call)
//   err      1 int                        device error word (zeroed per call)
//   experts  1 ExpertDev                  weight pointers of this call
//   strips   kMaxStrips + 1 ints          strip offsets
//   groups   kMaxStrips + 1 ints          column-slice offsets
constexpr size_t kOffLists = 0;
constexpr size_t kOffCounts = kOffLists + sizeof(int32_t) * pi::kMaxStrips * pi::kMaxStrip;
constexpr size_t kOffBar = (kOffCounts + sizeof(int32_t) * pi::kMaxStrips + 255) & ~size_t(255);
constexpr size_t kOffErr = kOffBar + sizeof(unsigned) * pi::kBarWords;
constexpr size_t kOffEx = (kOffErr + sizeof(int) + 255) & ~size_t(255);
constexpr size_t kOffStrips = kOffEx + sizeof(pi::ExpertDev);
constexpr size_t kOffGroups = kOffStrips + sizeof(int32_t) * (pi::kMaxStrips + 1);
constexpr size_t kNoAllocBytes = (kOffGroups + sizeof(int32_t) * (pi::kMaxStrips + 1) + 255) & ~size_t(255);

// Every device that loads the library holds this array until process exit.
// Every call shares it; a call leaves its contents behind.
static __device__ __align__(256) unsigned char g_pi_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_na_mutex;
unsigned char *g_na_ptr[kMaxDevices];    // device address of the array, per device

pi_status na_fail(pi_status st, const char *msg)
{
    char buf[256];
    snprintf(buf, sizeof buf, "pi_predict_noalloc: %s", msg);
    pi::set_last_error(buf);
    return st;
}

// Writes the call's tables into the array and clears what must start at zero
// (barrier words, error word); the count reads -1 until the
// predictor kernel completes.
__global__ void na_setup(unsigned char *base, const uint8_t *V, const uint8_t *U, const float *c,
                         int F, int S, int ng, int32_t *count)
{
    const int t = threadIdx.x;
    if (t == 0) {
        pi::ExpertDev *ex = reinterpret_cast<pi::ExpertDev *>(base + kOffEx);
        ex->V = V;
        ex->U = U;
        ex->c = c;
        ex->Wgu = nullptr;
        ex->Wd = nullptr;
        ex->sU = nullptr;
        ex->sV = nullptr;
        ex->Wgu_cold = nullptr;
        ex->Wd_cold = nullptr;
    }
    int32_t *strips = reinterpret_cast<int32_t *>(base + kOffStrips);
    int32_t *groups = reinterpret_cast<int32_t *>(base + kOffGroups);
    const int q = F / S, rem = F % S;
    for (int b = t; b <= S; b += blockDim.x) {
        strips[b] = b * q + (b < rem ? b : rem);
        groups[b] = int((long long)b * ng / S);
    }
    for (size_t i = t; i < (kOffEx - kOffBar) / 4; i += blockDim.x)
        reinterpret_cast<int *>(base + kOffBar)[i] = 0;
    if (t == 0) *count = -1;
}

// Runs after the predictor kernel on the same stream: a bounded wait that ran
// out in any CTA shows as *count = -1, whatever that CTA's peers wrote.
__global__ void na_finish(const int *err, int32_t *count)
{
    if (*reinterpret_cast<const volatile int *>(err) != 0) *count = -1;
}

}  // namespace

extern "C" PI_API pi_status pi_predict_noalloc(int d_model, int d_ff, int rank, pi_dtype pred_dtype,
                                               float threshold, const void *V_dev, const void *U_dev,
                                               const float *bias_dev, const float *x_dev,
                                               int32_t *idx_dev, int32_t *count_dev, float *z_dev,
                                               void *stream)
{
    if (!V_dev || !U_dev || !bias_dev || !x_dev || !idx_dev || !count_dev)
        return na_fail(PI_ERR_INVALID_ARG, "null argument");
    if (pred_dtype != PI_F32 && pred_dtype != PI_F16 && pred_dtype != PI_BF16)
        return na_fail(PI_ERR_INVALID_ARG, "pred_dtype must be F32, F16 or BF16");
    const int pb = pred_dtype == PI_F32 ? 4 : 2;
    if (d_model < 256 || d_model % 256 != 0 || d_model > (pb == 4 ? 4096 : 8192))
        return na_fail(PI_ERR_INVALID_ARG, "d_model must be a multiple of 256, <= 8192 (<= 4096 for F32)");
    if (rank < 1 || rank % 16 != 0 || rank > 128 * (16 / pb))
        return na_fail(PI_ERR_INVALID_ARG, "rank must be a multiple of 16 and <= 1024 (512 for F32)");
    if (!std::isfinite(threshold)) return na_fail(PI_ERR_INVALID_ARG, "threshold must be finite");
    const void *ptrs[] = {V_dev, U_dev, x_dev};
    for (const void *q : ptrs)
        if (reinterpret_cast<uintptr_t>(q) & 15u)
            return na_fail(PI_ERR_INVALID_ARG, "V, U and x must be 16-byte aligned");

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return na_fail(PI_ERR_CUDA, "no current CUDA device");
    if (dev >= kMaxDevices)
        return na_fail(PI_ERR_UNSUPPORTED, "the current device index is 64 or more (devices 0..63 supported)");
    int nsm = 0;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return na_fail(PI_ERR_CUDA, "cudaDeviceGetAttribute failed");
    const int fmt = pred_dtype == PI_F32 ? pi::kF32 : (pred_dtype == PI_F16 ? pi::kF16 : pi::kBF16);
    const int per_sm = pi::decode_max_blocks_per_sm(fmt, fmt, d_model);
    int S = nsm < pi::kMaxStrips ? nsm : pi::kMaxStrips;
    if (per_sm < 1) return na_fail(PI_ERR_UNSUPPORTED, "kernel does not fit on this device");
    if (d_ff < 1 || d_ff > pi::kMaxStrip * S)
        return na_fail(PI_ERR_INVALID_ARG, "d_ff must be in [1, 256 * min(SMs, 256)]");

    // One-time set-up per device (with that device current): the device
    // address of the static array.  Its name is only a host-side stand-in.
    unsigned char *base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_na_mutex);
        if (!g_na_ptr[dev]) {
            void *ptr = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&ptr, g_pi_noalloc_scratch);
            if (e != cudaSuccess) return na_fail(PI_ERR_CUDA, cudaGetErrorString(e));
            g_na_ptr[dev] = static_cast<unsigned char *>(ptr);
        }
        base = g_na_ptr[dev];
    }

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    na_setup<<<1, 256, 0, st>>>(base, static_cast<const uint8_t *>(V_dev), static_cast<const uint8_t *>(U_dev),
                                bias_dev, d_ff, S, d_model / 8, count_dev);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return na_fail(PI_ERR_CUDA, cudaGetErrorString(e));

    pi::DecodeParams p{};
    // One dense layer whose predictor is the caller's (V row-major, as the
    // decode kernel stores it); its FFN weights are never read.
    p.ex = reinterpret_cast<const pi::ExpertDev *>(base + kOffEx);
    p.router = nullptr;
    p.strip_off = reinterpret_cast<const int32_t *>(base + kOffStrips);
    p.grp_off = reinterpret_cast<const int32_t *>(base + kOffGroups);
    p.d = d_model;
    p.F = d_ff;
    p.r = rank;
    p.E = 1;
    p.top_k = 1;
    p.act = PI_ACT_REGLU;
    p.gated = 1;
    p.S = S;
    p.layer_begin = 0;
    p.layer_end = 1;
    p.threshold = threshold;
    p.eps = 1e-6f;
    p.vrow = d_model * pb;
    p.urow = rank * pb;
    p.wrow = d_model * pb;
    p.gu_bytes = 2 * p.wrow;
    p.spec_down = 0;
    p.rec_bytes = p.gu_bytes;
    p.wd_stride = p.wrow;
    p.u_swz = 0;          // the caller's U rows as they are
    p.mode = pi::kModePredict;
    p.pred_expert = 0;
    p.x_in = x_dev;
    p.z_out = z_dev;
    p.idx_out = idx_dev;
    p.count_out = count_dev;
    p.lists = reinterpret_cast<int32_t *>(base + kOffLists);
    p.counts = reinterpret_cast<int32_t *>(base + kOffCounts);
    p.bar = reinterpret_cast<unsigned *>(base + kOffBar);
    p.err = reinterpret_cast<int *>(base + kOffErr);
    p.wait_ns = 2000000000LL;
    p.debug_flags = 0;
    p.prof = nullptr;
    e = pi::launch_decode(fmt, fmt, p, st);
    if (e != cudaSuccess) return na_fail(PI_ERR_CUDA, cudaGetErrorString(e));
    na_finish<<<1, 1, 0, st>>>(p.err, count_dev);
    e = cudaGetLastError();
    if (e != cudaSuccess) return na_fail(PI_ERR_CUDA, cudaGetErrorString(e));
    return PI_OK;
}
