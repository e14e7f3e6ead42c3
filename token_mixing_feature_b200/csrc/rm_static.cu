// rm_pffn_forward_static: the per-token FFN without any device allocation.
//
// rm_pffn_forward needs a handle, and rm_create obtains the handle's workspace
// with cudaMalloc.  Some callers cannot allocate device memory at all -- code
// that runs where the CUDA allocator is off limits (inside another runtime's
// memory pool, or a host process whose device memory is fully reserved before
// this library is used).  For them this entry point keeps its one piece of
// scratch, the FFN hidden activations H [T, B, hidden], in a file-scope
// __device__ array of fixed size that every GPU loading the library holds
// until the process exits.  The caller passes only inputs and outputs.
//
// The array's name is only a host-side stand-in in host code: its device
// address is obtained once per device with cudaGetSymbolAddress (the first
// call on each device does this, with that device current) and then passed to
// the kernels.  All calls share the array, so calls that overlap on the GPU
// (different streams, or different host threads on one device) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "rm_internal.h"

namespace {

constexpr size_t kScratchBytes = RM_STATIC_SCRATCH_BYTES;
constexpr size_t kHiddenOffset = 256;   // [0, 8): device error word + site id
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_pffn_scratch[kScratchBytes];

std::mutex g_mu;
unsigned char* g_scratch_addr[kMaxDevices];

// Device address of g_pffn_scratch on the current device (looked up once).
rm_status scratch_address(unsigned char** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return RM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return RM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_pffn_scratch) != cudaSuccess || !p) return RM_ERR_CUDA;
        g_scratch_addr[dev] = static_cast<unsigned char*>(p);
    }
    *out = g_scratch_addr[dev];
    return RM_OK;
}

inline bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" rm_status rm_pffn_forward_static(const rm_block_weights* w, const void* S, void* V, int B, int T, int D,
                                            int hidden, rm_dtype dtype, int act, int* device_status,
                                            rm_stream_t stream) {
    if (!w || !aligned16(S) || !aligned16(V) || !aligned16(w->W1) || !aligned16(w->b1) || !aligned16(w->W2) ||
        !aligned16(w->b2))
        return RM_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || D < 1 || hidden < 1) return RM_ERR_INVALID_ARG;
    if (T > 64) return RM_ERR_UNSUPPORTED;   // the token limit of rm_create
    if (dtype != RM_BF16 && dtype != RM_F32) return RM_ERR_INVALID_ARG;
    if (act != RM_ACT_GELU_TANH && act != RM_ACT_GELU_ERF && act != RM_ACT_RELU) return RM_ERR_INVALID_ARG;
    if (dtype == RM_BF16 && (D % 16 || hidden % 16)) return RM_ERR_UNSUPPORTED;
    if (dtype == RM_F32 && (D % 4 || hidden % 4)) return RM_ERR_UNSUPPORTED;
    int dev = 0, num_sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return RM_ERR_CUDA;
    // H [T, B, hidden] must fit the array; each factor is checked against the
    // room left, so no product of the int arguments can wrap around.
    const size_t esz = dtype == RM_BF16 ? 2 : 4;
    const size_t room = kScratchBytes - kHiddenOffset;
    const size_t row = (size_t)hidden * esz;   // < 2^33, no wrap
    if (row > room || (size_t)B > room / row || (size_t)T > room / (row * (size_t)B))
        return RM_ERR_INVALID_ARG;

    unsigned char* scratch = nullptr;
    rm_status st = scratch_address(&scratch);
    if (st != RM_OK) return st;

    cudaStream_t s = stream;
    int* err_word = reinterpret_cast<int*>(scratch);
    // The array keeps the previous call's contents: the error word must start at zero.
    if (cudaMemsetAsync(err_word, 0, 2 * sizeof(int), s) != cudaSuccess) return RM_ERR_CUDA;
    void* H = scratch + kHiddenOffset;

    rm::GroupedGemm g1{};
    g1.G = T;
    g1.M = B;
    g1.N = hidden;
    g1.K = D;
    g1.A = S;
    g1.a_gstride = D;
    g1.a_ld = (long long)T * D;
    g1.W = w->W1;
    g1.out = H;
    g1.o_gstride = (long long)B * hidden;
    g1.o_ld = hidden;
    g1.bias = static_cast<const float*>(w->b1);
    g1.epi = rm::epi_for_act(act);

    rm::GroupedGemm g2{};
    g2.G = T;
    g2.M = B;
    g2.N = D;
    g2.K = hidden;
    g2.A = H;
    g2.a_gstride = (long long)B * hidden;
    g2.a_ld = hidden;
    g2.W = w->W2;
    g2.out = V;
    g2.o_gstride = D;
    g2.o_ld = (long long)T * D;
    g2.bias = static_cast<const float*>(w->b2);
    g2.epi = rm::EPI_BIAS_RESID;

    const rm::DeviceErr err{err_word, err_word + 1};
    const uint64_t budget_ns = 1000000000ull;
    cudaError_t e;
    if (dtype == RM_BF16) {
        e = rm::launch_gemm_tc(g1, err, budget_ns, num_sms, s);
        if (e == cudaSuccess) e = rm::launch_gemm_tc(g2, err, budget_ns, num_sms, s);
    } else {
        e = rm::launch_gemm_simt(g1, s);
        if (e == cudaSuccess) e = rm::launch_gemm_simt(g2, s);
    }
    if (e == cudaSuccess && device_status)
        e = cudaMemcpyAsync(device_status, err_word, sizeof(int), cudaMemcpyDeviceToDevice, s);
    return e == cudaSuccess ? RM_OK : RM_ERR_CUDA;
}
