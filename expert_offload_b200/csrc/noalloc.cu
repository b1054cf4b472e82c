// noalloc.cu - hfq4_moe_forward_noalloc: the single-layer routed-expert
// forward for callers that must not allocate device memory.
//
// Some callers cannot hand this library a workspace: code running while a
// framework captures a stream into a CUDA graph with its own allocator,
// serving loops that forbid any allocation after start-up, plugins whose host
// application gives them no allocator.  For them this entry point keeps its
// scratch (the persistent kernel's control words and the h buffer) in one
// file-scope device array, so a call allocates nothing.  The pages have no
// counterpart to this entry point.
#include <cstring>
#include <mutex>

#include "device.cuh"

namespace hfq {
namespace {

// Largest scratch the entry point supports: the control block plus h for
// T <= 8 tokens, k <= 16 experts per token and I <= 1024 (8*16*1024 floats).
constexpr size_t kNoAllocHBytes = (size_t)8 * 16 * 1024 * sizeof(float);
constexpr size_t kNoAllocCtlBytes = 36864;            // >= stack_ctl_bytes(), checked at run time
constexpr size_t kNoAllocBytes = kNoAllocCtlBytes + kNoAllocHBytes;

// Every device that loads this library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices];

// Device address of the array on the current device, resolved once per
// device (cudaGetSymbolAddress; the host-side name is only a stand-in).
hfq_status scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(HFQ_ERR_UNSUPPORTED, "device %d >= %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(HFQ_ERR_CUDA, "cudaGetSymbolAddress of the scratch array: %s",
                        cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return HFQ_OK;
}

}  // namespace

// hfq_workspace_status(NULL, 0, stream): the status word of this device's
// array.  HFQ_OK when no call has run on the device yet.  After an error the
// array's control block is cleared, as a workspace's would be.
hfq_status noalloc_status(cudaStream_t s)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> g(g_mu);
        if (dev >= 0 && dev < kMaxDevices) scratch = g_scratch_ptr[dev];
    }
    if (!scratch) return ok();
    unsigned word = 0;
    e = cudaMemcpyAsync(&word, scratch, sizeof word, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (word == 0) return ok();
    e = cudaMemsetAsync(scratch, 0, stack_ctl_bytes(), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "clearing the scratch: %s", cudaGetErrorString(e));
    const int st = (int)word;
    if (st == HFQ_ERR_ARG)
        return fail(HFQ_ERR_ARG, "the allocation-free forward found an invalid expert id (status %d)", st);
    return fail((hfq_status)st, "a device-side wait of the allocation-free forward ran out (status %d)", st);
}

}  // namespace hfq

using namespace hfq;

extern "C" hfq_status hfq4_moe_forward_noalloc(const hfq4_layer *layer, const void *x,
                                               hfq_dtype x_dtype, int T, const int32_t *idx,
                                               const float *wts, int k, float *y, void *y_bf16,
                                               void *stream)
{
    if (!layer || !layer->expert_ptr) return fail(HFQ_ERR_ARG, "layer or expert_ptr is null");
    hfq_status st = check_shape(layer->hidden, layer->inter, layer->n_experts, k);
    if (st) return st;
    if (!x || !idx || !wts || !y) return fail(HFQ_ERR_ARG, "hfq4_moe_forward_noalloc: null pointer");
    if (x_dtype != HFQ_F32 && x_dtype != HFQ_BF16) return fail(HFQ_ERR_ARG, "bad x_dtype");
    if (!aligned16(x) || !aligned16(y) || (y_bf16 && !aligned16(y_bf16)))
        return fail(HFQ_ERR_ALIGN, "x, y and y_bf16 must be 16-byte aligned");
    const size_t ip = (size_t)(layer->inter + HFQ4_BLOCK - 1) / HFQ4_BLOCK * HFQ4_BLOCK;
    const size_t need_h = (size_t)(T < 4 ? 4 : T) * k * ip * sizeof(float);
    if (T < 1 || T > 8 || k > 16 || layer->inter > 1024 || layer->hidden > 2048 ||
        need_h > kNoAllocHBytes || stack_ctl_bytes() > kNoAllocCtlBytes)
        return fail(HFQ_ERR_UNSUPPORTED,
                    "hfq4_moe_forward_noalloc takes T <= 8, k <= 16, inter <= 1024, hidden <= 2048 "
                    "(its fixed scratch is %zu bytes); got T=%d k=%d inter=%d hidden=%d", kNoAllocBytes,
                    T, k, layer->inter, layer->hidden);
    int sms = 0, dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "device query: %s", cudaGetErrorString(e));
    if (!stack_supported(T, layer->hidden, layer->inter, k, sms))
        return fail(HFQ_ERR_UNSUPPORTED, "hfq4_moe_forward_noalloc: shape (T=%d k=%d hidden=%d inter=%d) "
                    "not supported by the persistent kernel", T, k, layer->hidden, layer->inter);
    void *scratch = nullptr;
    if ((st = scratch_address(&scratch))) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // every call shares the array and finds the last call's contents in it:
    // the control words (the status word among them) must start at zero; the
    // launch epoch and layout signature after them are kept, so that the
    // one-token kernel's exchange tags never match h words an earlier call
    // left behind (a call with another k or inter clears h first)
    e = cudaMemsetAsync(scratch, 0, stack_ctl_clear_bytes(), s);
    if (e != cudaSuccess) return fail(HFQ_ERR_CUDA, "clearing the scratch: %s", cudaGetErrorString(e));
    float *h = reinterpret_cast<float *>(static_cast<char *>(scratch) + kNoAllocCtlBytes);
    st = launch_stack(layer, 1, nullptr, idx, wts, x, x_dtype == HFQ_F32, T, k, nullptr, nullptr, h,
                      y, static_cast<uint16_t *>(y_bf16), nullptr, nullptr,
                      static_cast<unsigned *>(scratch), option_wait_timeout_ns(),
                      option_take_extra_arrivals(), s);
    return st ? st : ok();
}
