// lb_linear_forward_noalloc: the decode forward of one layer with its scratch
// in a fixed static device array, for callers that must not allocate.
//
// The scratch lives in `g_noalloc_scratch` below.  In host code that name is
// only a host-side stand-in for the array, not a device address, so the host
// looks the real address up once per device (cudaGetSymbolAddress, with the
// device current) and passes that pointer on; device code in this file may
// name the array directly.

#include <mutex>

#include "lb_internal.cuh"

namespace lb {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LB_NOALLOC_SCRATCH_BYTES];

// Offsets inside the array.
constexpr size_t kOffDesc = 0;        // LayerDev (the kernels read descriptors from device memory)
constexpr size_t kOffMeta = 768;      // int2 [2][16]
constexpr size_t kOffAcc = 1024;      // double accumulators, then the fragments

static_assert(sizeof(LayerDev) <= 256, "descriptor slot");

constexpr int kMaxDevices = 64;
static void *g_addr[kMaxDevices];
static std::mutex g_addr_mu;

// Writes the descriptor and clears what the kernels expect to start at zero.
__global__ void noalloc_setup_kernel(LayerDev d, size_t acc_n)
{
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *reinterpret_cast<LayerDev *>(g_noalloc_scratch + kOffDesc) = d;
    }
    double *acc = reinterpret_cast<double *>(g_noalloc_scratch + kOffAcc);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < acc_n; i += (size_t)gridDim.x * blockDim.x)
        acc[i] = 0.0;
}

static size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }

}  // namespace lb

using namespace lb;

extern "C" lb_status lb_linear_forward_noalloc(const uint16_t *x, int M, const lb_layer *L, float *y, void *stream)
{
    set_launch_count(0);
    if (!L || M < 0) return LB_ERR_INVALID_ARG;
    if (M == 0) return LB_OK;
    if (!x || !y || ((uintptr_t)x & 15) || ((uintptr_t)y & 15)) return LB_ERR_INVALID_ARG;
    if (M > LB_DECODE_MAX_M) return LB_ERR_UNSUPPORTED;
    const LayerDev &src = L->d;
    const size_t acc_n = acc_doubles(src.R1);
    const size_t off_frag = kOffAcc + al256(acc_n * sizeof(double));
    const size_t off_xfrag = off_frag + al256((size_t)kMaxNT * src.KB2 * 32 * sizeof(uint2));
    const size_t off_xmeta = off_xfrag + al256((size_t)src.KB1e * 32 * sizeof(uint2));
    const size_t need = off_xmeta + (size_t)src.nkc * 4 * sizeof(int);
    if (need > LB_NOALLOC_SCRATCH_BYTES) return LB_ERR_UNSUPPORTED;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return status_from(e);
    if (dev < 0 || dev >= kMaxDevices) return LB_ERR_UNSUPPORTED;
    unsigned char *base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_addr_mu);
        if (!g_addr[dev]) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess) return status_from(e);
            g_addr[dev] = p;
        }
        base = static_cast<unsigned char *>(g_addr[dev]);
    }
    LayerDev d = src;
    d.acc = reinterpret_cast<double *>(base + kOffAcc);
    d.zfrag = reinterpret_cast<uint2 *>(base + off_frag);
    d.zmeta = reinterpret_cast<int2 *>(base + kOffMeta);
    d.xfrag = reinterpret_cast<uint2 *>(base + off_xfrag);
    d.xmeta = reinterpret_cast<int *>(base + off_xmeta);
    cudaStream_t s = (cudaStream_t)stream;
    noalloc_setup_kernel<<<64, 256, 0, s>>>(d, acc_n);
    if ((e = cudaGetLastError()) != cudaSuccess) return status_from(e);
    const Plan &P = L->self->plan;   // the layer's own work items (read only)
    int launches = 1;
    // a bounded wait that gives up reports to the layer's own error slot (allocated with the layer),
    // which lb_layer_status reads and clears
    lb_status st = decode_launch_one(reinterpret_cast<const LayerDev *>(base + kOffDesc), d, P, x, y, M, P.err, s,
                                     &launches);
    set_launch_count(launches);
    return st;
}
