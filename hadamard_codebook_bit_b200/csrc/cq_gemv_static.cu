// cq_gemv_static.cu -- cq_dequant_gemv for callers that cannot allocate device memory.
//
// The fused GEMV needs scratch space (the rotated activations in tensor-core fragment order,
// their exponents and a codeword table).  cq_dequant_gemv takes it from the caller; this
// entry point instead uses a fixed array in the library's own device memory, sized for
// cols <= kStaticMaxCols, so it never calls cudaMalloc / cudaFree or any allocating
// routine.  Every GPU that loads the library holds this array until the process exits.
#include <algorithm>
#include <cstdint>
#include <mutex>

#include "cq_internal.h"

namespace {

constexpr long long kStaticMaxCols = 32768;  // 256 groups of 128
constexpr int kChunk = 8;                      // activation rows per block (tensor-core N)
constexpr int kMaxBatch = 64;
constexpr long long kStaticMaxGroups = kStaticMaxCols / 128;
// 2080 bytes per group (8 k-steps x 32 lanes x 8 bytes of fp16 fragments + 8 fp32 exponents)
// plus the 48-byte codeword table, rounded up to 256 bytes.
constexpr size_t kStaticScratchBytes = ((kStaticMaxGroups * 2080 + 48 + 255) / 256) * 256;

// Shared by every call on a device: calls whose executions overlap on the GPU (e.g. issued to
// two streams without ordering between them) race on this array.
static __device__ __align__(256) unsigned char g_gemv_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];

// Device address of g_gemv_scratch on the current device (set up once per device).  In host
// code the symbol itself is only a host-side handle; the kernels need this address.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_gemv_scratch) != cudaSuccess || p == nullptr) return CQ_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return CQ_OK;
}

}  // namespace

extern "C" int cq_dequant_gemv_static(const unsigned char* packed, const unsigned short* norms,
                                      long long rows, long long cols, int bits, int group_size,
                                      const float* codebook, const void* x, int batch, float* y,
                                      void* stream) {
    if (cols > kStaticMaxCols) return CQ_ERR_WORKSPACE;  // beyond the built-in scratch
    if (batch < 1 || batch > kMaxBatch) return CQ_ERR_INVALID_ARG;
    const size_t need = cq_gemv_workspace_bytes(cols, std::min(batch, kChunk));
    if (need > kStaticScratchBytes) return CQ_ERR_WORKSPACE;
    // validate every argument (as the first block of rows would see it) before launching
    if (cols > 0 && rows > 0 && x == nullptr) return CQ_ERR_INVALID_ARG;
    void* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != CQ_OK) return rc;
    // The array holds one block of 8 activation rows, so larger batches run block after
    // block on `stream` (each block's rotation waits for the previous block's GEMV).  The
    // scratch needs no clearing: every call rewrites all of it that the kernels read.
    for (int c0 = 0; c0 < batch; c0 += kChunk) {
        const int b = std::min(kChunk, batch - c0);
        const void* xc = static_cast<const unsigned short*>(x) + static_cast<long long>(c0) * cols;
        rc = cq_dequant_gemv(packed, norms, rows, cols, bits, group_size, codebook,
                             x ? xc : nullptr, b, y ? y + static_cast<long long>(c0) * rows : nullptr,
                             scratch, kStaticScratchBytes, stream);
        if (rc != CQ_OK) return rc;
    }
    return CQ_OK;
}
