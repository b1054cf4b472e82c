// cache.cpp - dynamic VRAM expert cache over host-mapped experts, refilled by
// the copy engine, and the copy-engine staging of selected experts.
//
// Strata report, "model and engine": hot experts are kept in a VRAM cache in
// front of the pinned host arena (thousands of slots, hit rates of 96.9-99.5 %
// in its runs).  hipfire offload explainer, "PCIe pass-through": the kernels
// read host-mapped experts directly, with no staging copy.  Both live on the
// same per-layer pointer tables here: a table entry names an expert's HBM
// cache slot while it is cached, and its home address (HBM, or the device
// alias of its pinned host bytes) otherwise; the kernels read whatever the
// table names.  The cache only moves bytes (cudaMemcpyAsync from pinned
// memory, i.e. the copy engine) and rewrites table entries, in stream order.
#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "common.h"

struct hfq_cache {
    int L = 0, E = 0, slots = 0;
    size_t eb = 0;
    uint8_t *slot_mem = nullptr;           // device: [L][slots] expert slots
    uint64_t *table_dev = nullptr;         // device [L][E] pointer tables (null: bookkeeping only)
    uint8_t *loc_dev = nullptr;            // device [L][E] locations, or null
    std::vector<uint64_t> home, host_src;  // [L][E]
    std::vector<uint8_t> home_loc;         // [L][E]: 1 = home is host memory
    std::vector<int> slot_of;              // [L][E]: cache slot, or -1
    std::vector<int> owner;                // [L][slots]: expert, or -1
    std::vector<float> freq;               // [L][E] selection frequency
    std::vector<uint32_t> nobs;            // [L] observations
    // pinned staging of the tables: [L][2][E] pointers, [L][2][E] locations,
    // and per layer an event after the last copy that read its staging
    uint64_t *stage_ptr = nullptr;
    uint8_t *stage_loc = nullptr;
    std::vector<cudaEvent_t> staged;       // [L]
    std::vector<char> staged_live;         // [L]: the event was recorded
    // refills (max_admit >= 0 with device tables) copy on their own stream and
    // name their slots in the layer's next call: [L] admissions in flight, the
    // events after the layer's evicting table write and after its copies
    cudaStream_t copy_stream = nullptr;
    std::vector<std::vector<std::pair<int, int>>> pending;
    std::vector<cudaEvent_t> evicted_ev, copied_ev;
    std::vector<int> pending_slot;         // [L][E]: slot of an admission in flight, or -1
    uint64_t hits = 0, misses = 0, admitted = 0, evicted = 0;
};

namespace {

constexpr uint32_t kHalveEvery = 256;      // observations of a layer between halvings of its frequencies

uint64_t table_entry(const hfq_cache *c, int l, int e)
{
    const size_t i = (size_t)l * c->E + e;
    const int s = c->slot_of[i];
    return s >= 0 ? reinterpret_cast<uint64_t>(c->slot_mem + ((size_t)l * c->slots + s) * c->eb) : c->home[i];
}

uint8_t loc_entry(const hfq_cache *c, int l, int e)
{
    const size_t i = (size_t)l * c->E + e;
    return c->slot_of[i] >= 0 ? 0 : c->home_loc[i];
}

// Layer l's tables (as the bookkeeping says now) into its staging buffer `b`,
// then to the device.
hfq_status write_tables(hfq_cache *c, int l, int b, cudaStream_t s)
{
    uint64_t *p = c->stage_ptr + ((size_t)l * 2 + b) * c->E;
    uint8_t *q = c->stage_loc + ((size_t)l * 2 + b) * c->E;
    for (int e = 0; e < c->E; ++e) {
        p[e] = table_entry(c, l, e);
        q[e] = loc_entry(c, l, e);
    }
    cudaError_t err = cudaMemcpyAsync(c->table_dev + (size_t)l * c->E, p, (size_t)c->E * 8,
                                      cudaMemcpyHostToDevice, s);
    if (err == cudaSuccess && c->loc_dev)
        err = cudaMemcpyAsync(c->loc_dev + (size_t)l * c->E, q, (size_t)c->E, cudaMemcpyHostToDevice, s);
    if (err != cudaSuccess) return hfq::fail(HFQ_ERR_CUDA, "cache table write: %s", cudaGetErrorString(err));
    return HFQ_OK;
}

// The layer's admissions in flight name their slots: the tables are written
// behind their copies (the compute stream waits for the copy stream).
hfq_status commit_pending(hfq_cache *c, int l, cudaStream_t s)
{
    auto &pend = c->pending[l];
    if (pend.empty()) return HFQ_OK;
    cudaError_t err = cudaStreamWaitEvent(s, c->copied_ev[l], 0);
    if (err != cudaSuccess) return hfq::fail(HFQ_ERR_CUDA, "cache commit: %s", cudaGetErrorString(err));
    const size_t base = (size_t)l * c->E;
    for (auto &a : pend) {
        c->slot_of[base + a.first] = a.second;
        c->pending_slot[base + a.first] = -1;
    }
    c->admitted += pend.size();
    pend.clear();
    return write_tables(c, l, 1, s);
}

}  // namespace

using namespace hfq;

extern "C" {

hfq_status hfq_cache_create(int L, int E, size_t expert_bytes, int slots, const uint64_t *home,
                            const uint64_t *host_src, const uint8_t *home_loc, void *slot_mem,
                            size_t slot_bytes, uint64_t *table_dev, uint8_t *loc_dev, void *stream,
                            hfq_cache **out)
{
    if (!out || L < 1 || L > HFQ_MAX_STACK_LAYERS || E < 1 || E > HFQ_MAX_EXPERTS || slots < 0 ||
        slots > E || !expert_bytes || !home || !host_src || !home_loc)
        return fail(HFQ_ERR_ARG, "hfq_cache_create: bad argument");
    if (table_dev) {
        if (slots && (!slot_mem || slot_bytes < (size_t)L * slots * expert_bytes))
            return fail(HFQ_ERR_ARG, "hfq_cache_create: slot memory of %zu bytes needed, %zu given",
                        (size_t)L * slots * expert_bytes, slot_bytes);
        if ((slot_mem && !aligned16(slot_mem)) || expert_bytes % 16 || !aligned16(table_dev))
            return fail(HFQ_ERR_ALIGN, "hfq_cache_create: slots and tables must be 16-byte aligned");
    }
    for (size_t i = 0; i < (size_t)L * E; ++i)
        if (home_loc[i] && !host_src[i])
            return fail(HFQ_ERR_ARG, "hfq_cache_create: host expert %zu has no host address", i);
    hfq_cache *c = new (std::nothrow) hfq_cache;
    if (!c) return fail(HFQ_ERR_ALLOC, "hfq_cache_create: out of host memory");
    c->L = L; c->E = E; c->slots = slots; c->eb = expert_bytes;
    c->slot_mem = static_cast<uint8_t *>(slot_mem);
    c->table_dev = table_dev;
    c->loc_dev = loc_dev;
    const size_t n = (size_t)L * E;
    c->home.assign(home, home + n);
    c->host_src.assign(host_src, host_src + n);
    c->home_loc.assign(home_loc, home_loc + n);
    c->slot_of.assign(n, -1);
    c->owner.assign((size_t)L * slots, -1);
    c->freq.assign(n, 0.0f);
    c->nobs.assign(L, 0);
    if (table_dev) {
        void *p = nullptr, *q = nullptr;
        cudaError_t err = cudaHostAlloc(&p, (size_t)L * 2 * E * 8, cudaHostAllocDefault);
        if (err == cudaSuccess) err = cudaHostAlloc(&q, (size_t)L * 2 * E, cudaHostAllocDefault);
        if (err != cudaSuccess) {
            if (p) cudaFreeHost(p);
            delete c;
            return fail(HFQ_ERR_ALLOC, "hfq_cache_create: pinned staging of %zu bytes: %s",
                        (size_t)L * 2 * E * 9, cudaGetErrorString(err));
        }
        c->stage_ptr = static_cast<uint64_t *>(p);
        c->stage_loc = static_cast<uint8_t *>(q);
        c->staged.assign(L, nullptr);
        c->staged_live.assign(L, 0);
        c->evicted_ev.assign(L, nullptr);
        c->copied_ev.assign(L, nullptr);
        c->pending.assign(L, {});
        c->pending_slot.assign(n, -1);
        for (int l = 0; l < L && err == cudaSuccess; ++l) {
            err = cudaEventCreateWithFlags(&c->staged[l], cudaEventDisableTiming);
            if (err == cudaSuccess) err = cudaEventCreateWithFlags(&c->evicted_ev[l], cudaEventDisableTiming);
            if (err == cudaSuccess) err = cudaEventCreateWithFlags(&c->copied_ev[l], cudaEventDisableTiming);
        }
        if (err == cudaSuccess) err = cudaStreamCreateWithFlags(&c->copy_stream, cudaStreamNonBlocking);
        if (err != cudaSuccess) {
            hfq_cache_destroy(c);
            return fail(HFQ_ERR_CUDA, "hfq_cache_create: events: %s", cudaGetErrorString(err));
        }
        // nothing cached yet: every table names the experts' homes
        cudaStream_t s = (cudaStream_t)stream;
        for (int l = 0; l < L; ++l) {
            hfq_status st = write_tables(c, l, 0, s);
            if (st == HFQ_OK && cudaStreamSynchronize(s) != cudaSuccess)
                st = fail(HFQ_ERR_CUDA, "hfq_cache_create: table write");
            if (st != HFQ_OK) {
                hfq_cache_destroy(c);
                return st;
            }
        }
    }
    *out = c;
    return ok();
}

hfq_status hfq_cache_observe(hfq_cache *c, int layer, const int32_t *ids, int n, int max_admit, void *stream)
{
    if (!c || layer < 0 || layer >= c->L || n < 0 || (n && !ids))
        return fail(HFQ_ERR_ARG, "hfq_cache_observe: bad argument");
    for (int i = 0; i < n; ++i)
        if (ids[i] < 0 || ids[i] >= c->E)
            return fail(HFQ_ERR_ARG, "hfq_cache_observe: expert id %d outside [0, %d)", ids[i], c->E);
    cudaStream_t s = (cudaStream_t)stream;
    // the layer's staging buffers are rewritten below: the copies that read
    // them in the layer's previous call must have run (nothing else on the
    // stream is waited for)
    if (c->table_dev && c->staged_live[layer]) {
        const cudaError_t err = cudaEventSynchronize(c->staged[layer]);
        if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "hfq_cache_observe: %s", cudaGetErrorString(err));
        c->staged_live[layer] = 0;
    }
    const int E = c->E;
    const size_t base = (size_t)layer * E;
    hfq_status st = HFQ_OK;
    // the previous call's refills name their slots from the next kernel on
    bool wrote = false;
    if (c->table_dev && !c->pending[layer].empty()) {
        if ((st = commit_pending(c, layer, s)) != HFQ_OK) return st;
        wrote = true;
    }
    std::vector<int> cand;                 // missed host experts, once each
    std::vector<char> selected(E, 0);
    for (int i = 0; i < n; ++i) {
        const int e = ids[i];
        c->freq[base + e] += 1.0f;
        if (selected[e]) continue;
        selected[e] = 1;
        if (!c->home_loc[base + e] || c->slot_of[base + e] >= 0) {
            ++c->hits;
        } else if (c->table_dev && c->pending_slot[base + e] >= 0) {
            ++c->misses;                               // its copy is in flight
        } else {
            ++c->misses;
            cand.push_back(e);
        }
    }
    if (++c->nobs[layer] % kHalveEvery == 0)
        for (int e = 0; e < E; ++e) c->freq[base + e] *= 0.5f;
    // most frequent first, ties to the lower expert
    std::sort(cand.begin(), cand.end(), [&](int x, int y) {
        const float fx = c->freq[base + x], fy = c->freq[base + y];
        return fx != fy ? fx > fy : x < y;
    });
    int *owner = c->owner.data() + (size_t)layer * c->slots;
    std::vector<std::pair<int, int>> admits;    // (expert, slot)
    bool any_evict = false;
    const size_t limit = max_admit < 0 ? cand.size() : std::min(cand.size(), (size_t)max_admit);
    for (size_t i = 0; i < limit; ++i) {
        const int e = cand[i];
        int slot = -1;
        for (int q = 0; q < c->slots && slot < 0; ++q)
            if (owner[q] < 0) slot = q;
        if (slot < 0) {
            // the least frequent cached expert not selected in this call
            int victim = -1;
            for (int q = 0; q < c->slots; ++q) {
                const int v = owner[q];
                if (v < 0 || selected[v] || (c->table_dev && c->pending_slot[base + v] >= 0)) continue;
                if (victim < 0 || c->freq[base + v] < c->freq[base + owner[victim]] ||
                    (c->freq[base + v] == c->freq[base + owner[victim]] && v < owner[victim]))
                    victim = q;
            }
            if (victim < 0) break;                       // every slot holds an expert of this call
            if (max_admit >= 0 && !(c->freq[base + e] > c->freq[base + owner[victim]])) break;
            c->slot_of[base + owner[victim]] = -1;
            owner[victim] = -1;
            ++c->evicted;
            any_evict = true;
            slot = victim;
        }
        owner[slot] = e;
        admits.emplace_back(e, slot);
    }
    if (!c->table_dev) {                                 // bookkeeping only
        for (auto &a : admits) c->slot_of[base + a.first] = a.second;
        c->admitted += admits.size();
        return ok();
    }
    auto record_staged = [&]() -> hfq_status {
        const cudaError_t err = cudaEventRecord(c->staged[layer], s);
        if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "hfq_cache_observe: event: %s", cudaGetErrorString(err));
        c->staged_live[layer] = 1;
        return HFQ_OK;
    };
    if (!any_evict && admits.empty()) {
        if (wrote && (st = record_staged()) != HFQ_OK) return st;
        return ok();
    }
    // 1. evicted experts back home (the admitted ones still read from home)
    if (any_evict && (st = write_tables(c, layer, 0, s)) != HFQ_OK) return st;
    if (max_admit >= 0) {
        // refill: the copies run on the cache's copy stream once the kernels
        // enqueued so far (which may read the victims' slots) are done; the
        // slots are named in the layer's next call
        cudaError_t err = cudaEventRecord(c->evicted_ev[layer], s);
        if (err == cudaSuccess) err = cudaStreamWaitEvent(c->copy_stream, c->evicted_ev[layer], 0);
        for (size_t i = 0; i < admits.size() && err == cudaSuccess; ++i) {
            const auto &a = admits[i];
            void *dst = c->slot_mem + ((size_t)layer * c->slots + a.second) * c->eb;
            err = cudaMemcpyAsync(dst, reinterpret_cast<const void *>(c->host_src[base + a.first]), c->eb,
                                  cudaMemcpyHostToDevice, c->copy_stream);
            c->pending_slot[base + a.first] = a.second;
        }
        if (err == cudaSuccess) err = cudaEventRecord(c->copied_ev[layer], c->copy_stream);
        if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "hfq_cache_observe: refill: %s", cudaGetErrorString(err));
        c->pending[layer] = admits;
        if ((st = record_staged()) != HFQ_OK) return st;
        return ok();
    }
    // 2. the admitted experts' bytes into their slots (copy engine)
    for (auto &a : admits) {
        void *dst = c->slot_mem + ((size_t)layer * c->slots + a.second) * c->eb;
        const cudaError_t err = cudaMemcpyAsync(dst, reinterpret_cast<const void *>(c->host_src[base + a.first]),
                                                c->eb, cudaMemcpyHostToDevice, s);
        if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "hfq_cache_observe: copy: %s", cudaGetErrorString(err));
    }
    // 3. then the admitted experts' entries name their slots
    for (auto &a : admits) c->slot_of[base + a.first] = a.second;
    c->admitted += admits.size();
    if (!admits.empty() && (st = write_tables(c, layer, 1, s)) != HFQ_OK) return st;
    if ((st = record_staged()) != HFQ_OK) return st;
    return ok();
}

hfq_status hfq_cache_flush(hfq_cache *c, void *stream)
{
    if (!c) return fail(HFQ_ERR_ARG, "hfq_cache_flush: no cache");
    if (!c->table_dev) return ok();
    cudaStream_t s = (cudaStream_t)stream;
    for (int l = 0; l < c->L; ++l) {
        if (c->pending[l].empty()) continue;
        if (c->staged_live[l]) {
            const cudaError_t err = cudaEventSynchronize(c->staged[l]);
            if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "hfq_cache_flush: %s", cudaGetErrorString(err));
            c->staged_live[l] = 0;
        }
        hfq_status st = commit_pending(c, l, s);
        if (st != HFQ_OK) return st;
        const cudaError_t err = cudaEventRecord(c->staged[l], s);
        if (err != cudaSuccess) return fail(HFQ_ERR_CUDA, "hfq_cache_flush: event: %s", cudaGetErrorString(err));
        c->staged_live[l] = 1;
    }
    return ok();
}

hfq_status hfq_cache_slot_of(const hfq_cache *c, int layer, int expert, int *slot)
{
    if (!c || !slot || layer < 0 || layer >= c->L || expert < 0 || expert >= c->E)
        return fail(HFQ_ERR_ARG, "hfq_cache_slot_of: bad argument");
    *slot = c->slot_of[(size_t)layer * c->E + expert];
    return ok();
}

hfq_status hfq_cache_stats(const hfq_cache *c, uint64_t *hits, uint64_t *misses, uint64_t *admitted,
                           uint64_t *evicted)
{
    if (!c) return fail(HFQ_ERR_ARG, "hfq_cache_stats: no cache");
    if (hits) *hits = c->hits;
    if (misses) *misses = c->misses;
    if (admitted) *admitted = c->admitted;
    if (evicted) *evicted = c->evicted;
    return ok();
}

hfq_status hfq_cache_destroy(hfq_cache *c)
{
    if (!c) return fail(HFQ_ERR_ARG, "hfq_cache_destroy: no cache");
    // pending copies still read the staging buffers or write the slots
    if (c->copy_stream) {
        cudaStreamSynchronize(c->copy_stream);
        cudaStreamDestroy(c->copy_stream);
    }
    for (size_t l = 0; l < c->staged.size(); ++l) {
        if (c->staged[l]) {
            if (c->staged_live[l]) cudaEventSynchronize(c->staged[l]);
            cudaEventDestroy(c->staged[l]);
        }
        if (c->evicted_ev[l]) cudaEventDestroy(c->evicted_ev[l]);
        if (c->copied_ev[l]) cudaEventDestroy(c->copied_ev[l]);
    }
    if (c->stage_ptr) cudaFreeHost(c->stage_ptr);
    if (c->stage_loc) cudaFreeHost(c->stage_loc);
    delete c;
    return ok();
}

}  // extern "C"
