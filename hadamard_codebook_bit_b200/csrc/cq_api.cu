// cq_api.cu -- the extern "C" entry points of libcq (declared in include/cq.h).
//
// Host side only: argument validation (before any launch), the per-device default
// codebook, and dispatch to the kernel launchers.  Nothing here computes on the data.
#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include <vector>

#include "cq_internal.h"

namespace cq {

namespace {

constexpr int kMaxDevices = 64;

// Default codebooks live in device memory of every GPU that used them: slot 0 = ternary,
// 1 = 2-bit, 2 = 3-bit, 3 = 4-bit.  Filled lazily, once per (device, slot).
__device__ float g_default_codebooks[4][16];

// Watchdog status of the kernels on this device (bit 0: a bounded wait gave up).
__device__ unsigned g_status;

std::mutex g_mu;
bool g_default_ready[kMaxDevices][4];
int g_sm_count[kMaxDevices];
unsigned* g_status_ptr[kMaxDevices];

int slot_for_bits(int bits) { return bits == CQ_BITS_TERNARY ? 0 : bits - 1; }

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

// Device pointer of the default codebook for `bits` on the current device, uploading it on
// first use (synchronous copy).
cudaError_t default_codebook(int bits, const float** out) {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const int slot = slot_for_bits(bits);
    std::lock_guard<std::mutex> lock(g_mu);
    void* base = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&base, g_default_codebooks);
    if (e != cudaSuccess) return e;
    float* dst = static_cast<float*>(base) + 16 * slot;
    if (!g_default_ready[dev][slot]) {
        float host[16] = {0};
        if (host_codebook(bits, kGroup, 0, host) < 0) return cudaErrorInvalidValue;
        e = cudaMemcpy(dst, host, sizeof(host), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return e;
        g_default_ready[dev][slot] = true;
    }
    *out = dst;
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool bits_ok(int bits) { return bits == CQ_BITS_TERNARY || (bits >= 2 && bits <= 4); }

int check_common(long long rows, long long cols, int bits, int group_size) {
    if (rows < 0 || cols < 0 || !bits_ok(bits)) return CQ_ERR_INVALID_ARG;
    if (group_size <= 0 || (group_size & (group_size - 1))) return CQ_ERR_INVALID_ARG;
    if (group_size != kGroup) return CQ_ERR_UNSUPPORTED;
    // keep every byte offset well inside 64-bit arithmetic
    if (cols > 0 && rows > (1LL << 40) / cols) return CQ_ERR_INVALID_ARG;
    return CQ_OK;
}

Shape make_shape(long long rows, long long cols) {
    Shape s;
    s.rows = rows;
    s.cols = cols;
    s.groups_per_row = (cols + kGroup - 1) / kGroup;
    s.total_groups = rows * s.groups_per_row;
    return s;
}

int resolve_codebook(int bits, const float* codebook, const float** cb) {
    if (codebook != nullptr) {
        if ((reinterpret_cast<uintptr_t>(codebook) & 3u) != 0) return CQ_ERR_ALIGNMENT;
        *cb = codebook;
        return CQ_OK;
    }
    return default_codebook(bits, cb) == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

// Activation rows per GEMV launch job (the tensor-core B operand holds 8 batch columns).
// Larger batches, up to kMaxGemvBatch, become ceil(batch / 8) jobs of the same launch pair,
// one per block of 8 rows of x and y, each with its own slice of the caller's workspace.
constexpr int kGemvChunk = 8;
constexpr int kMaxGemvBatch = 64;

void push_gemv_chunks(std::vector<GemvItem>& items, const unsigned char* packed,
                      const unsigned short* norms, long long rows, long long cols, const void* x,
                      int batch, float* y, void* workspace) {
    const size_t chunk_ws = gemv_workspace_bytes(cols, kGemvChunk);
    const Shape sh = make_shape(rows, cols);
    for (int c0 = 0; c0 < batch; c0 += kGemvChunk) {
        items.push_back({packed, norms, sh, static_cast<const uint16_t*>(x) + static_cast<long long>(c0) * cols,
                         std::min(kGemvChunk, batch - c0), y + static_cast<long long>(c0) * rows,
                         static_cast<char*>(workspace) + static_cast<size_t>(c0 / kGemvChunk) * chunk_ws});
    }
}

}  // namespace

bool is_default_codebook(int bits, const float* cb) {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices || !bits_ok(bits)) return false;
    const int slot = slot_for_bits(bits);
    void* base = nullptr;
    if (cudaGetSymbolAddress(&base, g_default_codebooks) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(g_mu);
    return g_default_ready[dev][slot] && cb == static_cast<const float*>(base) + 16 * slot;
}

unsigned* device_status_ptr() {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_status_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<unsigned*>(p);
    }
    return g_status_ptr[dev];
}

EncodeTiledFn tensor_map_encoder() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool tcgen05_enabled() {
    static const bool on = [] {
        const char* v = std::getenv("CQ_DISABLE_TCGEN05");
        return v == nullptr || v[0] == '\0' || (v[0] == '0' && v[1] == '\0');
    }();
    return on;
}

int sm_count() {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_sm_count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

}  // namespace cq

extern "C" {

const char* cq_status_string(int status) {
    switch (status) {
        case CQ_OK: return "CQ_OK";
        case CQ_ERR_INVALID_ARG: return "CQ_ERR_INVALID_ARG: invalid argument";
        case CQ_ERR_UNSUPPORTED: return "CQ_ERR_UNSUPPORTED: valid but not implemented (group_size must be 128)";
        case CQ_ERR_CUDA: return "CQ_ERR_CUDA: a CUDA call or kernel launch failed";
        case CQ_ERR_ALIGNMENT: return "CQ_ERR_ALIGNMENT: device pointer not 16-byte aligned";
        case CQ_ERR_WORKSPACE: return "CQ_ERR_WORKSPACE: workspace missing or too small";
        default: return "CQ: unknown status";
    }
}

int cq_version(void) { return 10000; }

int cq_device_status(int reset, unsigned* status_out) {
    if (status_out == nullptr) return CQ_ERR_INVALID_ARG;
    unsigned* p = cq::device_status_ptr();
    if (p == nullptr) return CQ_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return CQ_ERR_CUDA;
    if (reset) {
        const unsigned zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return CQ_ERR_CUDA;
    }
    *status_out = v;
    return CQ_OK;
}

int cq_codebook(int bits, int group_size, unsigned long long seed, float* out_host, int* n_levels) {
    if (out_host == nullptr || seed > 0xffffffffULL) return CQ_ERR_INVALID_ARG;
    const int L = cq::host_codebook(bits, group_size, seed, out_host);
    if (L < 0) return CQ_ERR_INVALID_ARG;
    if (n_levels) *n_levels = L;
    return CQ_OK;
}

size_t cq_packed_bytes(long long rows, long long cols, int bits, int group_size) {
    const int fb = cq::field_bits_for(bits);
    if (rows < 0 || cols < 0 || fb < 0 || group_size < 8 || (group_size & (group_size - 1)))
        return 0;
    const long long G = (cols + group_size - 1) / group_size;
    return static_cast<size_t>(rows) * static_cast<size_t>(G) *
           static_cast<size_t>(group_size * fb / 8);
}

size_t cq_norm_bytes(long long rows, long long cols, int group_size) {
    if (rows < 0 || cols < 0 || group_size < 8 || (group_size & (group_size - 1))) return 0;
    const long long G = (cols + group_size - 1) / group_size;
    return 2 * static_cast<size_t>(rows) * static_cast<size_t>(G);
}

int cq_quantize(const void* w, int w_dtype, long long rows, long long cols, int bits,
                int group_size, const float* codebook, unsigned char* packed_out,
                unsigned short* norms_out, void* stream) {
    if (w_dtype != CQ_F32 && w_dtype != CQ_BF16) return CQ_ERR_INVALID_ARG;
    int rc = cq::check_common(rows, cols, bits, group_size);
    if (rc != CQ_OK) return rc;
    if (rows == 0 || cols == 0) return CQ_OK;  // nothing to quantise
    if (!w || !packed_out || !norms_out) return CQ_ERR_INVALID_ARG;
    if (!cq::aligned16(w) || !cq::aligned16(packed_out) || !cq::aligned16(norms_out))
        return CQ_ERR_ALIGNMENT;
    const float* cb = nullptr;
    rc = cq::resolve_codebook(bits, codebook, &cb);
    if (rc != CQ_OK) return rc;
    const cudaError_t e = cq::launch_quantize(w, w_dtype, cq::make_shape(rows, cols), bits, cb,
                                              packed_out, norms_out,
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

int cq_dequantize(const unsigned char* packed, const unsigned short* norms, long long rows,
                  long long cols, int bits, int group_size, const float* codebook, void* out,
                  int out_dtype, void* stream) {
    if (out_dtype != CQ_F32 && out_dtype != CQ_BF16) return CQ_ERR_INVALID_ARG;
    int rc = cq::check_common(rows, cols, bits, group_size);
    if (rc != CQ_OK) return rc;
    if (rows == 0 || cols == 0) return CQ_OK;  // nothing to write
    if (!packed || !norms || !out) return CQ_ERR_INVALID_ARG;
    if (!cq::aligned16(packed) || !cq::aligned16(norms) || !cq::aligned16(out))
        return CQ_ERR_ALIGNMENT;
    const float* cb = nullptr;
    rc = cq::resolve_codebook(bits, codebook, &cb);
    if (rc != CQ_OK) return rc;
    const cudaError_t e = cq::launch_dequantize(packed, norms, cq::make_shape(rows, cols), bits,
                                                cb, out, out_dtype,
                                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

int cq_quantize_batch(const cq_quantize_job* jobs, int count, int w_dtype, int bits,
                      int group_size, const float* codebook, void* stream) {
    if (count < 0 || (count > 0 && !jobs)) return CQ_ERR_INVALID_ARG;
    if (w_dtype != CQ_F32 && w_dtype != CQ_BF16) return CQ_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) {
        const cq_quantize_job& j = jobs[i];
        const int rc = cq::check_common(j.rows, j.cols, bits, group_size);
        if (rc != CQ_OK) return rc;
        if (j.rows == 0 || j.cols == 0) continue;
        if (!j.w || !j.packed_out || !j.norms_out) return CQ_ERR_INVALID_ARG;
        if (!cq::aligned16(j.w) || !cq::aligned16(j.packed_out) || !cq::aligned16(j.norms_out))
            return CQ_ERR_ALIGNMENT;
    }
    bool any = false;
    for (int i = 0; i < count; ++i) any = any || (jobs[i].rows > 0 && jobs[i].cols > 0);
    if (!any) return CQ_OK;  // nothing to quantise
    const float* cb = nullptr;
    int rc = cq::resolve_codebook(bits, codebook, &cb);
    if (rc != CQ_OK) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::vector<cq::QuantizeItem> tc;
    unsigned* status = cq::device_status_ptr();
    for (int i = 0; i < count; ++i) {
        const cq_quantize_job& j = jobs[i];
        if (j.rows == 0 || j.cols == 0) continue;
        const cq::Shape sh = cq::make_shape(j.rows, j.cols);
        if (status && cq::tcgen05_enabled() && cq::quantize_tc_supported(w_dtype, sh)) {
            tc.push_back({j.w, sh, j.packed_out, j.norms_out});
        } else {
            const cudaError_t e = cq::launch_quantize(j.w, w_dtype, sh, bits, cb, j.packed_out, j.norms_out, st);
            if (e != cudaSuccess) return CQ_ERR_CUDA;
        }
    }
    if (!tc.empty()) {
        const cudaError_t e = cq::launch_quantize_tc_batch(tc.data(), static_cast<int>(tc.size()), bits, cb, status, st);
        if (e != cudaSuccess) return CQ_ERR_CUDA;
    }
    return CQ_OK;
}

int cq_dequantize_batch(const cq_dequantize_job* jobs, int count, int bits, int group_size,
                        const float* codebook, int out_dtype, void* stream) {
    if (count < 0 || (count > 0 && !jobs)) return CQ_ERR_INVALID_ARG;
    if (out_dtype != CQ_F32 && out_dtype != CQ_BF16) return CQ_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) {
        const cq_dequantize_job& j = jobs[i];
        const int rc = cq::check_common(j.rows, j.cols, bits, group_size);
        if (rc != CQ_OK) return rc;
        if (j.rows == 0 || j.cols == 0) continue;
        if (!j.packed || !j.norms || !j.out) return CQ_ERR_INVALID_ARG;
        if (!cq::aligned16(j.packed) || !cq::aligned16(j.norms) || !cq::aligned16(j.out))
            return CQ_ERR_ALIGNMENT;
    }
    bool any = false;
    for (int i = 0; i < count; ++i) any = any || (jobs[i].rows > 0 && jobs[i].cols > 0);
    if (!any) return CQ_OK;  // nothing to write
    const float* cb = nullptr;
    int rc = cq::resolve_codebook(bits, codebook, &cb);
    if (rc != CQ_OK) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::vector<cq::DequantizeItem> tc;
    unsigned* status = cq::device_status_ptr();
    for (int i = 0; i < count; ++i) {
        const cq_dequantize_job& j = jobs[i];
        if (j.rows == 0 || j.cols == 0) continue;
        const cq::Shape sh = cq::make_shape(j.rows, j.cols);
        if (status && cq::tcgen05_enabled() && cq::dequantize_tc_supported(out_dtype, sh)) {
            tc.push_back({j.packed, j.norms, sh, j.out});
        } else {
            const cudaError_t e = cq::launch_dequantize(j.packed, j.norms, sh, bits, cb, j.out, out_dtype, st);
            if (e != cudaSuccess) return CQ_ERR_CUDA;
        }
    }
    if (!tc.empty()) {
        const cudaError_t e = cq::launch_dequantize_tc_batch(tc.data(), static_cast<int>(tc.size()), bits, cb,
                                                             out_dtype, status, st);
        if (e != cudaSuccess) return CQ_ERR_CUDA;
    }
    return CQ_OK;
}

int cq_fake_quantize(const void* w, int w_dtype, long long rows, long long cols, int bits,
                     int group_size, const float* codebook, unsigned char* packed_out,
                     unsigned short* norms_out, void* out, int out_dtype, void* stream) {
    // Validate what the dequantise step adds before the quantise step launches anything.
    if (out_dtype != CQ_F32 && out_dtype != CQ_BF16) return CQ_ERR_INVALID_ARG;
    if (w_dtype != CQ_F32 && w_dtype != CQ_BF16) return CQ_ERR_INVALID_ARG;
    const int rc = cq::check_common(rows, cols, bits, group_size);
    if (rc != CQ_OK) return rc;
    if (rows == 0 || cols == 0) return CQ_OK;
    if (!out) return CQ_ERR_INVALID_ARG;
    if (!cq::aligned16(out)) return CQ_ERR_ALIGNMENT;
    const cq_fake_quantize_job job = {w, rows, cols, packed_out, norms_out, out};
    return cq_fake_quantize_batch(&job, 1, w_dtype, bits, group_size, codebook, out_dtype, stream);
}

int cq_fake_quantize_batch(const cq_fake_quantize_job* jobs, int count, int w_dtype, int bits,
                           int group_size, const float* codebook, int out_dtype, void* stream) {
    if (count < 0 || (count > 0 && !jobs)) return CQ_ERR_INVALID_ARG;
    if (w_dtype != CQ_F32 && w_dtype != CQ_BF16) return CQ_ERR_INVALID_ARG;
    if (out_dtype != CQ_F32 && out_dtype != CQ_BF16) return CQ_ERR_INVALID_ARG;
    std::vector<cq_quantize_job> q;
    std::vector<cq_dequantize_job> d;
    q.reserve(static_cast<size_t>(count));
    d.reserve(static_cast<size_t>(count));
    for (int i = 0; i < count; ++i) {
        const cq_fake_quantize_job& j = jobs[i];
        const int rc = cq::check_common(j.rows, j.cols, bits, group_size);
        if (rc != CQ_OK) return rc;
        if (j.rows == 0 || j.cols == 0) continue;
        if (!j.w || !j.packed_out || !j.norms_out || !j.out) return CQ_ERR_INVALID_ARG;
        if (!cq::aligned16(j.w) || !cq::aligned16(j.packed_out) || !cq::aligned16(j.norms_out) ||
            !cq::aligned16(j.out))
            return CQ_ERR_ALIGNMENT;
        q.push_back({j.w, j.rows, j.cols, j.packed_out, j.norms_out});
        d.push_back({j.packed_out, j.norms_out, j.rows, j.cols, j.out});
    }
    if (q.empty()) return CQ_OK;
    if (codebook != nullptr && (reinterpret_cast<uintptr_t>(codebook) & 3u) != 0) return CQ_ERR_ALIGNMENT;
    // Both steps now pass their own validation; only a CUDA failure can stop the second.
    const int rc = cq_quantize_batch(q.data(), static_cast<int>(q.size()), w_dtype, bits, group_size,
                                     codebook, stream);
    if (rc != CQ_OK) return rc;
    return cq_dequantize_batch(d.data(), static_cast<int>(d.size()), bits, group_size, codebook,
                               out_dtype, stream);
}

int cq_dequant_gemv_batch(const cq_gemv_job* jobs, int count, int bits, int group_size,
                          const float* codebook, void* stream) {
    if (count < 0 || (count > 0 && !jobs)) return CQ_ERR_INVALID_ARG;
    bool any = false;
    for (int i = 0; i < count; ++i) {
        const cq_gemv_job& j = jobs[i];
        if (j.batch < 1 || j.batch > cq::kMaxGemvBatch) return CQ_ERR_INVALID_ARG;
        const int rc = cq::check_common(j.rows, j.cols, bits, group_size);
        if (rc != CQ_OK) return rc;
        if (j.rows == 0) continue;
        if (!j.y) return CQ_ERR_INVALID_ARG;
        if (!cq::aligned16(j.y)) return CQ_ERR_ALIGNMENT;
        any = true;
        if (j.cols == 0) continue;
        if (!j.packed || !j.norms || !j.x) return CQ_ERR_INVALID_ARG;
        if (!j.workspace || j.workspace_bytes < cq::gemv_workspace_bytes(j.cols, j.batch))
            return CQ_ERR_WORKSPACE;
        if (!cq::aligned16(j.packed) || !cq::aligned16(j.norms) || !cq::aligned16(j.x) ||
            !cq::aligned16(j.workspace))
            return CQ_ERR_ALIGNMENT;
    }
    if (!any) return CQ_OK;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::vector<cq::GemvItem> items;
    for (int i = 0; i < count; ++i) {
        const cq_gemv_job& j = jobs[i];
        if (j.rows == 0) continue;
        if (j.cols == 0) {  // empty inner dimension: y = 0
            const cudaError_t e = cudaMemsetAsync(j.y, 0, sizeof(float) * static_cast<size_t>(j.batch) *
                                                              static_cast<size_t>(j.rows), st);
            if (e != cudaSuccess) return CQ_ERR_CUDA;
            continue;
        }
        cq::push_gemv_chunks(items, j.packed, j.norms, j.rows, j.cols, j.x, j.batch, j.y, j.workspace);
    }
    if (items.empty()) return CQ_OK;
    const float* cb = nullptr;
    const int rc = cq::resolve_codebook(bits, codebook, &cb);
    if (rc != CQ_OK) return rc;
    const cudaError_t e = cq::launch_dequant_gemv_batch(items.data(), static_cast<int>(items.size()), bits, cb, st);
    return e == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

size_t cq_gemv_workspace_bytes(long long cols, int batch) {
    if (cols < 0 || batch < 1 || batch > cq::kMaxGemvBatch) return 0;
    return cq::gemv_workspace_bytes(cols, batch);
}

int cq_dequant_gemv(const unsigned char* packed, const unsigned short* norms, long long rows,
                    long long cols, int bits, int group_size, const float* codebook,
                    const void* x, int batch, float* y, void* workspace,
                    size_t workspace_bytes, void* stream) {
    if (batch < 1 || batch > cq::kMaxGemvBatch) return CQ_ERR_INVALID_ARG;
    int rc = cq::check_common(rows, cols, bits, group_size);
    if (rc != CQ_OK) return rc;
    if (rows == 0) return CQ_OK;  // y is empty
    if (!y) return CQ_ERR_INVALID_ARG;
    if (!cq::aligned16(y)) return CQ_ERR_ALIGNMENT;
    if (cols == 0) {  // empty inner dimension: y = 0
        const cudaError_t e = cudaMemsetAsync(y, 0, sizeof(float) * static_cast<size_t>(batch) *
                                                        static_cast<size_t>(rows),
                                              static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
    }
    if (!packed || !norms || !x) return CQ_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < cq::gemv_workspace_bytes(cols, batch))
        return CQ_ERR_WORKSPACE;
    if (!cq::aligned16(packed) || !cq::aligned16(norms) || !cq::aligned16(x) ||
        !cq::aligned16(y) || !cq::aligned16(workspace))
        return CQ_ERR_ALIGNMENT;
    const float* cb = nullptr;
    rc = cq::resolve_codebook(bits, codebook, &cb);
    if (rc != CQ_OK) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (batch > cq::kGemvChunk) {  // one launch pair over the blocks of 8 activation rows
        std::vector<cq::GemvItem> items;
        cq::push_gemv_chunks(items, packed, norms, rows, cols, x, batch, y, workspace);
        const cudaError_t e = cq::launch_dequant_gemv_batch(items.data(), static_cast<int>(items.size()), bits, cb, st);
        return e == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
    }
    const cudaError_t e = cq::launch_dequant_gemv(
        packed, norms, cq::make_shape(rows, cols), bits, cb, static_cast<const uint16_t*>(x),
        batch, y, workspace, st);
    return e == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

}  // extern "C"
