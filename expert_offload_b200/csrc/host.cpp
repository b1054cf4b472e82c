// host.cpp - host-only parts of libhfq4moe: error strings, sizes, the host
// HFQ4 packer, expert placement and the pinned host arena.
#include <sys/mman.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>
#include <algorithm>

#include <cuda_runtime.h>

#include "common.h"

namespace hfq {

static thread_local char g_msg[512];

hfq_status fail(hfq_status st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

hfq_status ok()
{
    g_msg[0] = 0;
    return HFQ_OK;
}

hfq_status check_shape(int hidden, int inter, int n_experts, int k)
{
    if (hidden <= 0 || inter <= 0 || hidden % 128 || inter % 128 || hidden > 8192 || inter > 8192)
        return fail(HFQ_ERR_UNSUPPORTED, "hidden=%d inter=%d: both must be multiples of 128 in "
                    "[128, 8192]", hidden, inter);
    if (n_experts < 1 || n_experts > HFQ_MAX_EXPERTS)
        return fail(HFQ_ERR_UNSUPPORTED, "n_experts=%d outside [1, %d]", n_experts, HFQ_MAX_EXPERTS);
    if (k < 1 || k > HFQ_MAX_TOPK || k > n_experts)
        return fail(HFQ_ERR_UNSUPPORTED, "k=%d outside [1, min(%d, E=%d)]", k, HFQ_MAX_TOPK, n_experts);
    return HFQ_OK;
}

// ---------------------------------------------------------------- packing
//
// One block of the HFQ4 format (hipfire thread, "HFQ quantisation format and
// GEMV"): min/max over the real elements, 15 steps, nearest-even rounding,
// f32 arithmetic throughout (this file is built with -ffp-contract=off, so
// no multiply-add is fused).
static void pack_block(const float *w, int n, uint8_t *out)
{
    float mn = w[0], mx = w[0];
    for (int i = 1; i < n; ++i) {
        mn = w[i] < mn ? w[i] : mn;
        mx = w[i] > mx ? w[i] : mx;
    }
    volatile float range = mx - mn;          // one f32 rounding
    float scale = range / 15.0f;             // one f32 rounding
    float zero = mn;
    std::memcpy(out, &scale, 4);
    std::memcpy(out + 4, &zero, 4);
    uint8_t *nib = out + 8;
    std::memset(nib, 0, 128);
    if (scale == 0.0f) return;
    for (int i = 0; i < n; ++i) {
        volatile float d = w[i] - zero;
        float t = d / scale;
        float r = std::nearbyint(t);         // default rounding mode: to nearest even
        int q = r < 0.0f ? 0 : (r > 15.0f ? 15 : (int)r);
        nib[i >> 1] |= (uint8_t)(q << ((i & 1) * 4));
    }
}

static void pack_matrix(const float *w, int rows, int cols, uint8_t *out)
{
    size_t nb = blocks_per_row(cols);
    for (int r = 0; r < rows; ++r)
        for (size_t b = 0; b < nb; ++b) {
            int c0 = (int)(b * HFQ4_BLOCK);
            int n = std::min(HFQ4_BLOCK, cols - c0);
            pack_block(w + (size_t)r * cols + c0, n, out + ((size_t)r * nb + b) * HFQ4_BLOCK_BYTES);
        }
}

}  // namespace hfq

using namespace hfq;

extern "C" {

const char *hfq_last_error(void) { return g_msg; }

int hfq_version(void) { return 10000; }

size_t hfq4_matrix_bytes(int rows, int cols)
{
    if (rows <= 0 || cols <= 0) return 0;
    return matrix_bytes(rows, cols);
}

size_t hfq4_expert_bytes(int hidden, int inter)
{
    if (hidden <= 0 || inter <= 0) return 0;
    return expert_bytes(hidden, inter);
}

hfq_status hfq4_pack_experts(const float *gate, const float *up, const float *down,
                             int n_experts, int hidden, int inter, void *out, size_t out_bytes)
{
    if (!gate || !up || !down || !out) return fail(HFQ_ERR_ARG, "hfq4_pack_experts: null pointer");
    if (n_experts < 1 || hidden < 1 || inter < 1)
        return fail(HFQ_ERR_ARG, "hfq4_pack_experts: n_experts=%d hidden=%d inter=%d", n_experts,
                    hidden, inter);
    size_t eb = expert_bytes(hidden, inter);
    if (out_bytes < eb * (size_t)n_experts)
        return fail(HFQ_ERR_ARG, "hfq4_pack_experts: out_bytes=%zu < %zu needed", out_bytes,
                    eb * (size_t)n_experts);
    size_t gsz = (size_t)inter * hidden, dsz = (size_t)hidden * inter;
    size_t mg = matrix_bytes(inter, hidden);
    for (int e = 0; e < n_experts; ++e) {
        uint8_t *o = static_cast<uint8_t *>(out) + eb * e;
        pack_matrix(gate + gsz * e, inter, hidden, o);
        pack_matrix(up + gsz * e, inter, hidden, o + mg);
        pack_matrix(down + dsz * e, hidden, inter, o + 2 * mg);
    }
    return ok();
}

// ---------------------------------------------------------------- placement
//
// hipfire offload explainer, "placement algorithm": first N layers resident
// (or auto fit-capacity), hot set of each host layer resident, loud refusal.

hfq_status hfq_placement_build(int L, int E, size_t eb, const uint32_t *counts,
                               int resident_layers, int hot_per_layer, size_t hbm_budget,
                               uint8_t *loc_out, int64_t *slot_out, size_t *hbm_needed,
                               size_t *host_needed)
{
    if (L < 1 || E < 1 || eb == 0 || !counts || !loc_out || !slot_out || !hbm_needed ||
        !host_needed)
        return fail(HFQ_ERR_ARG, "hfq_placement_build: bad argument");
    if (resident_layers > L || resident_layers < -1)
        return fail(HFQ_ERR_ARG, "hfq_placement_build: resident_layers=%d not in [-1, L=%d]",
                    resident_layers, L);
    size_t h = (size_t)std::max(0, std::min(hot_per_layer, E));
    auto need = [&](int n) { return ((size_t)n * E + (size_t)(L - n) * h) * eb; };
    int n = resident_layers;
    if (n < 0) {
        for (int c = L; c >= 0 && n < 0; --c)
            if (need(c) <= hbm_budget) n = c;
        if (n < 0) {
            *hbm_needed = need(0);
            *host_needed = (size_t)L * E * eb - need(0);
            return fail(HFQ_ERR_NOFIT, "DOES NOT FIT: hot sets alone need %zu bytes of HBM, budget "
                        "%zu, deficit %zu bytes; fix: raise the budget or lower hot_per_layer",
                        need(0), hbm_budget, need(0) - hbm_budget);
        }
    }
    std::vector<int> order(E);
    for (int l = 0; l < L; ++l) {
        uint8_t *loc = loc_out + (size_t)l * E;
        if (l < n) {
            std::fill(loc, loc + E, 0);
            continue;
        }
        std::fill(loc, loc + E, 1);
        const uint32_t *c = counts + (size_t)l * E;
        for (int e = 0; e < E; ++e) order[e] = e;
        std::stable_sort(order.begin(), order.end(),
                         [&](int a, int b) { return c[a] > c[b]; });   // stable: lower index first
        for (size_t i = 0; i < h; ++i) loc[order[i]] = 0;
    }
    int64_t next[2] = {0, 0};
    for (size_t i = 0; i < (size_t)L * E; ++i) slot_out[i] = next[loc_out[i]]++;
    *hbm_needed = (size_t)next[0] * eb;
    *host_needed = (size_t)next[1] * eb;
    if (*hbm_needed > hbm_budget)
        return fail(HFQ_ERR_NOFIT, "DOES NOT FIT: experts need %zu bytes of HBM with %d resident "
                    "layers and %zu hot experts per host layer, budget %zu, deficit %zu bytes; "
                    "fix: lower resident_layers or raise the budget", *hbm_needed, n, h,
                    hbm_budget, *hbm_needed - hbm_budget);
    return ok();
}

hfq_status hfq_placement_pointers(int L, int E, size_t eb, const uint8_t *loc, const int64_t *slot,
                                  const void *hbm_base, const void *host_dev_base, uint64_t *out)
{
    if (L < 1 || E < 1 || !loc || !slot || !out) return fail(HFQ_ERR_ARG, "bad argument");
    for (size_t i = 0; i < (size_t)L * E; ++i) {
        const void *base = loc[i] ? host_dev_base : hbm_base;
        if (!base) return fail(HFQ_ERR_ARG, "no base address for location %d", (int)loc[i]);
        out[i] = (uint64_t)(uintptr_t)base + (uint64_t)slot[i] * eb;
    }
    return ok();
}

// ---------------------------------------------------------------- host arena
//
// Strata report, pitfall 7: the pinned expert arena is registered with the
// CUDA runtime (portable), with 2 MiB pages only when the system gives them.

namespace {
struct Arena {
    void *host;
    size_t bytes;
    bool mmapped;
};
std::mutex g_arena_mu;
std::vector<Arena> g_arenas;
}  // namespace

hfq_status hfq_host_arena_create(size_t bytes, int flags, void **host, void **dev)
{
    if (!bytes || !host || !dev) return fail(HFQ_ERR_ARG, "hfq_host_arena_create: bad argument");
    void *p = nullptr;
    bool mm = false;
    cudaError_t err;
    if (flags & HFQ_ARENA_HUGEPAGE) {
        size_t two_mib = (size_t)2 << 20;
        size_t len = (bytes + two_mib - 1) / two_mib * two_mib;
        p = mmap(nullptr, len, PROT_READ | PROT_WRITE, MAP_PRIVATE | MAP_ANONYMOUS, -1, 0);
        if (p == MAP_FAILED)
            return fail(HFQ_ERR_ALLOC, "mmap of %zu bytes for the expert arena failed", len);
        madvise(p, len, MADV_HUGEPAGE);   // a hint; 4 KiB pages otherwise
        err = cudaHostRegister(p, len, cudaHostRegisterMapped | cudaHostRegisterPortable);
        if (err != cudaSuccess) {
            munmap(p, len);
            return fail(HFQ_ERR_ALLOC, "cudaHostRegister of %zu bytes failed: %s", len,
                        cudaGetErrorString(err));
        }
        bytes = len;
        mm = true;
    } else {
        err = cudaHostAlloc(&p, bytes, cudaHostAllocMapped | cudaHostAllocPortable);
        if (err != cudaSuccess)
            return fail(HFQ_ERR_ALLOC, "cudaHostAlloc of %zu pinned bytes failed: %s", bytes,
                        cudaGetErrorString(err));
    }
    void *d = nullptr;
    err = cudaHostGetDevicePointer(&d, p, 0);
    if (err != cudaSuccess) {
        if (mm) { cudaHostUnregister(p); munmap(p, bytes); } else cudaFreeHost(p);
        return fail(HFQ_ERR_ALLOC, "cudaHostGetDevicePointer failed: %s", cudaGetErrorString(err));
    }
    {
        std::lock_guard<std::mutex> g(g_arena_mu);
        g_arenas.push_back({p, bytes, mm});
    }
    *host = p;
    *dev = d;
    return ok();
}

hfq_status hfq_host_arena_destroy(void *host)
{
    Arena a{};
    {
        std::lock_guard<std::mutex> g(g_arena_mu);
        auto it = std::find_if(g_arenas.begin(), g_arenas.end(),
                               [&](const Arena &x) { return x.host == host; });
        if (it == g_arenas.end()) return fail(HFQ_ERR_ARG, "not an arena of this library");
        a = *it;
        g_arenas.erase(it);
    }
    if (a.mmapped) {
        cudaHostUnregister(a.host);
        munmap(a.host, a.bytes);
    } else {
        cudaFreeHost(a.host);
    }
    return ok();
}

}  // extern "C"
