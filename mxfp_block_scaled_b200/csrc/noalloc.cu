// noalloc.cu -- the verifier for callers that cannot allocate device memory.
//
// mxq_dequant_relerr needs a caller-provided workspace for its per-chunk
// partial sums.  Some callers cannot provide one: engines that reserve
// their whole device-memory budget up front for their own pools and forbid
// any further cudaMalloc, and host code paths that must not risk the
// device-wide synchronisation a cudaMalloc / cudaFree can cause.  For them,
// mxq_dequant_relerr_noalloc keeps the partial sums in a fixed array that is
// part of this library's device image instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it (kScratchBytes) until the process exits.  In host code
// its name only stands for the variable: the device address is obtained
// with cudaGetSymbolAddress, with that device current, once per device and
// context (set-up on the first call, and again after the device's context
// was replaced, e.g. by cudaDeviceReset, whose new context places the array
// anew), and cached here.
#include "mxq.h"
#include "mxq_internal.h"

#include <cuda.h>
#include <mutex>

namespace {

constexpr size_t kScratchBytes = size_t(2) << 20;   // 2 MiB: 131072 chunk partials
constexpr int kMaxDevices = 128;

static __device__ __align__(256) unsigned char g_verify_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};   // context the address belongs to

// Unique id of the calling thread's current context (0 when there is none
// or the driver cannot tell), through the driver entry points the runtime
// hands out, so the library needs no link-time dependency on the driver.
unsigned long long current_context_id()
{
    typedef CUresult (*GetCurrent)(CUcontext *);
    typedef CUresult (*GetId)(CUcontext, unsigned long long *);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {                                   // under g_mu
        void *f1 = nullptr, *f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<GetCurrent>(f1);
            get_id = reinterpret_cast<GetId>(f2);
        }
        (void)cudaGetLastError();
        resolved = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_verify_scratch on the current device: looked up on
// the first call for that device and whenever its context differs from the
// one the cached address was looked up in (or cannot be identified).
mxq_status scratch_for_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return MXQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices)
        return MXQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    const unsigned long long ctx = current_context_id();
    if (!g_scratch_addr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_verify_scratch) != cudaSuccess || !p)
            return MXQ_ERR_CUDA;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = current_context_id();   // the lookup made the context current
    }
    *out = g_scratch_addr[dev];
    return MXQ_OK;
}

} // namespace

extern "C" mxq_status mxq_dequant_relerr_noalloc(const uint16_t *x, const uint8_t *codes,
                                                 const uint8_t *scales, const float *s2,
                                                 mxq_fmt fmt, int64_t n_tensors, int64_t rows,
                                                 int64_t cols, int64_t tensors_per_scale,
                                                 double *sum_sq_err, double *sum_sq_ref,
                                                 double *relerr, cudaStream_t stream)
{
    // Requests that need more partial sums than the array holds are refused
    // by the size check of mxq_dequant_relerr (MXQ_ERR_WORKSPACE) before
    // anything is enqueued.  No partial sum needs to start at zero: each call
    // writes every partial it later reads.
    void *scratch = nullptr;
    const mxq_status st = scratch_for_current_device(&scratch);
    if (st != MXQ_OK)
        return st;
    return mxq_dequant_relerr(x, codes, scales, s2, fmt, MXQ_LAYOUT_LINEAR, n_tensors, rows, cols,
                              tensors_per_scale,
                              sum_sq_err, sum_sq_ref, relerr, scratch, kScratchBytes, stream);
}
