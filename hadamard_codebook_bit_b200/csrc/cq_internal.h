// cq_internal.h -- declarations shared by the C-ABI layer and the kernel files of libcq.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>  // CUtensorMap and its enums (types only; no libcuda link)
#include <cuda_runtime.h>

#include "cq.h"

namespace cq {

constexpr int kGroup = 128;

int levels_for_bits(int bits);
int field_bits_for(int bits);
int host_codebook(int bits, int group_size, unsigned long long seed, float* out);
// True when cb is the default codebook for `bits` on the current device (uploaded already).
bool is_default_codebook(int bits, const float* cb);

// Number of SMs of the current device (cached per device).
int sm_count();

// Shape of one quantised matrix as the kernels see it.
struct Shape {
    long long rows;
    long long cols;
    long long groups_per_row;  // G = ceil(cols / 128)
    long long total_groups;    // rows * G
};

// Launch with programmatic stream serialization: the kernel may start while the previous
// kernel in the stream is still running (after that kernel's griddepcontrol.launch_dependents).
// Every kernel of this library therefore executes griddepcontrol.wait before its first global
// memory access (read or write); only on-chip set-up (shared memory tables, barriers, tensor
// memory) runs earlier.  Kernels that follow in the stream without this attribute still wait
// for full completion.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Kernel launchers (one per file).  All return cudaSuccess or the launch error.
// cuTensorMapEncodeTiled, looked up once through the runtime's driver entry point (nullptr
// when unavailable).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

// Device-wide status word of the current device (bit 0: a bounded wait inside a kernel gave
// up).  Returns nullptr if the symbol address cannot be obtained.
unsigned* device_status_ptr();

// True when the tensor-core (tcgen05 + TMA) implementations are enabled for this process
// (environment variable CQ_DISABLE_TCGEN05 unset or "0").
bool tcgen05_enabled();

// One tensor of a batched call.
struct QuantizeItem {
    const void* w;
    Shape sh;
    uint8_t* packed;
    uint16_t* norms;
};
struct DequantizeItem {
    const uint8_t* packed;
    const uint16_t* norms;
    Shape sh;
    void* out;
};

struct GemvItem {
    const uint8_t* packed;
    const uint16_t* norms;
    Shape sh;
    const uint16_t* x;
    int batch;
    float* y;
    void* workspace;
};

// Tensor-core quantiser (cq_quantize_tc.cu): bf16 input, cols % 8 == 0.
bool quantize_tc_supported(int w_dtype, const Shape& s);
cudaError_t launch_quantize_tc(const void* w, const Shape& s, int bits, const float* codebook,
                               uint8_t* packed, uint16_t* norms, unsigned* status,
                               cudaStream_t stream);
// Several tensors (each quantize_tc_supported, none empty) in as few launches as possible.
cudaError_t launch_quantize_tc_batch(const QuantizeItem* items, int count, int bits,
                                     const float* codebook, unsigned* status, cudaStream_t stream);

// Tensor-core dequantiser (cq_dequantize_tc.cu): rows of the output start on 16 bytes.
bool dequantize_tc_supported(int out_dtype, const Shape& s);
cudaError_t launch_dequantize_tc(const uint8_t* packed, const uint16_t* norms, const Shape& s,
                                 int bits, const float* codebook, void* out, int out_dtype,
                                 unsigned* status, cudaStream_t stream);
// Several tensors (each dequantize_tc_supported, none empty) in as few launches as possible.
cudaError_t launch_dequantize_tc_batch(const DequantizeItem* items, int count, int bits,
                                       const float* codebook, int out_dtype, unsigned* status,
                                       cudaStream_t stream);

cudaError_t launch_quantize(const void* w, int w_dtype, const Shape& s, int bits,
                            const float* codebook, uint8_t* packed, uint16_t* norms,
                            cudaStream_t stream);
cudaError_t launch_dequantize(const uint8_t* packed, const uint16_t* norms, const Shape& s,
                              int bits, const float* codebook, void* out, int out_dtype,
                              cudaStream_t stream);
size_t gemv_workspace_bytes(long long cols, int batch);
cudaError_t launch_dequant_gemv(const uint8_t* packed, const uint16_t* norms, const Shape& s,
                                int bits, const float* codebook, const uint16_t* x, int batch,
                                float* y, void* workspace, cudaStream_t stream);
// Several products (none with rows == 0 or cols == 0) in as few launches as possible.
cudaError_t launch_dequant_gemv_batch(const GemvItem* items, int count, int bits,
                                      const float* codebook, cudaStream_t stream);

}  // namespace cq
