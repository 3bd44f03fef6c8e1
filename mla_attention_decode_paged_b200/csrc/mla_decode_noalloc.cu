// mla_decode_noalloc.cu -- mla_decode for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: a plugin running inside another runtime that
// owns all device memory and forbids allocation on its execution path, or a latency
// critical path where cudaMalloc's implicit device-wide synchronisation is not
// acceptable.  They still own q, the cache, the block table, seq_lens, out and lse, but
// they cannot hand the library a workspace.  This entry point uses a scratch array
// compiled into the library instead: a file-scope __device__ array of a fixed size,
// which every GPU that loads the library holds until the process exits.
//
// In host code the array's name is only a host-side stand-in, never a device address,
// so its device address is looked up with cudaGetSymbolAddress (with the caller's device
// current) and passed to the kernels like any workspace pointer.
#include <mutex>

#include "mla_decode_params.cuh"

namespace {

constexpr size_t kScratchBytes = (size_t)MLA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxCachedDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxCachedDevices] = {};

// Device address of g_scratch on the current device.  Outside stream capture it is looked
// up on every call (cudaGetSymbolAddress allocates nothing), so a context that was reset
// and reloaded the module never gets a stale address.  Inside a capture the lookup is not
// made; the address cached by the last call outside capture is used instead.
mla_status scratch_address(cudaStream_t stream, void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return MLA_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return MLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (cap != cudaStreamCaptureStatusNone) {
        if (dev >= kMaxCachedDevices || g_scratch_addr[dev] == nullptr) return MLA_ERR_CUDA;
        *out = g_scratch_addr[dev];
        return MLA_OK;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
    if (dev < kMaxCachedDevices) g_scratch_addr[dev] = p;
    *out = p;
    return MLA_OK;
}

}  // namespace

extern "C" mla_status mla_decode_noalloc(const void* q, const void* kv_pages, int kv_dtype, float kv_scale,
                                         const int32_t* block_table, int max_pages_per_req,
                                         const int32_t* seq_lens, int B, int s_q, int H, int64_t num_pages,
                                         float scale, int causal, void* out, float* lse, void* stream) {
    if (!q || !kv_pages || !block_table || !seq_lens || !out || !lse) return MLA_ERR_INVALID_ARG;
    if (B <= 0 || s_q <= 0 || H <= 0) return MLA_ERR_INVALID_ARG;
    if ((int64_t)s_q * H > mla::kMaxRows) return MLA_ERR_UNSUPPORTED;
    const int sms = mla::effective_sms();
    if (sms <= 0) return MLA_ERR_CUDA;
    const mla::WsLayout L = mla::make_layout(B, s_q, H, mla::num_groups_for(sms, mla::num_row_blocks(s_q, H)));
    if ((size_t)L.total > kScratchBytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
    void* ws = nullptr;
    mla_status st = scratch_address((cudaStream_t)stream, &ws);
    if (st != MLA_OK) return st;
    // The plan rewrites the whole header, the status word included, so nothing left in
    // the scratch by an earlier call is read before it is written again.
    st = mla_decode_plan(seq_lens, B, s_q, H, sms, ws, kScratchBytes, stream);
    if (st != MLA_OK) return st;
    return mla_decode(q, kv_pages, kv_dtype, kv_scale, block_table, max_pages_per_req, seq_lens, B, s_q, H,
                      num_pages, scale, causal, ws, kScratchBytes, out, lse, stream);
}
