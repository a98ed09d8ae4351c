// pages.cpp -- host page allocator for the paged KV pools (include/pkv_pages.h):
// block tables, per-page reference counts and a free-list stack, kept in
// host memory between decode steps of a continuous-batching loop.  Pages are
// handed out on demand as positions cross a page boundary and return to the
// pool as soon as their last request releases them ("TensorRT-LLM Guide:
// High-Throughput GPU Inference Engine", sections "1. In-Flight Batching:
// Continuous Iteration Scheduling" and "2. Paged KV Cache & Memory
// Virtualization").  No exception crosses the C ABI: every allocation here
// happens in pkv_pages_create, and nothing else throws.
#include <stdlib.h>
#include <string.h>

#include <new>
#include <utility>
#include <vector>

#include "../../include/pkv_pages.h"

struct pkv_pages {
    int num_pages, P, max_batch, max_blocks;
    std::vector<int32_t> table;      // [max_batch][max_blocks], -1 past a slot's pages
    std::vector<int32_t> lens;       // [max_batch] tokens in the cache
    std::vector<int32_t> active;     // [max_batch] 0 / 1
    std::vector<int32_t> npages;     // [max_batch] pages in the slot's row
    std::vector<int32_t> ref;        // [num_pages] reference counts
    std::vector<int32_t> free_stack; // free page ids; the top is handed out first
    int free_top = 0;                // entries of free_stack in use
    std::vector<int32_t> log;        // (slot, index, value) of every table write since the last take
    bool log_full = false;           // more writes than the log holds: the caller must copy the table
    std::vector<uint8_t> seen;       // [max_batch][max_blocks] scratch of pkv_pages_take_changes, all 0 between calls
};

namespace {

int pages_for(long long tokens, int P) { return (int)((tokens + P - 1) / P); }

void set_entry(pkv_pages* pp, int slot, int i, int32_t value)
{
    pp->table[(size_t)slot * pp->max_blocks + i] = value;
    if (pp->log_full) return;
    if (pp->log.size() + 3 > pp->log.capacity()) {   // never reallocates: past capacity, a full copy is due
        pp->log_full = true;
        return;
    }
    pp->log.push_back(slot);
    pp->log.push_back(i);
    pp->log.push_back(value);
}

int32_t pop_page(pkv_pages* pp)
{
    const int32_t page = pp->free_stack[--pp->free_top];
    pp->ref[page] = 1;
    return page;
}

void drop_page(pkv_pages* pp, int32_t page)
{
    if (--pp->ref[page] == 0) pp->free_stack[pp->free_top++] = page;
}

bool slot_ok(const pkv_pages* pp, int slot) { return pp && slot >= 0 && slot < pp->max_batch; }

}  // namespace

extern "C" {

pkv_status pkv_pages_create(int num_pages, int page_size, int max_batch, int max_blocks_per_seq, pkv_pages** out)
{
    if (!out || num_pages <= 0 || page_size <= 0 || max_batch <= 0 || max_blocks_per_seq <= 0)
        return PKV_ERR_INVALID_ARG;
    if ((long long)max_batch * max_blocks_per_seq > (1LL << 31) - 1) return PKV_ERR_INVALID_ARG;
    pkv_pages* pp = new (std::nothrow) pkv_pages;
    if (!pp) return PKV_ERR_OOM;
    try {
        pp->num_pages = num_pages;
        pp->P = page_size;
        pp->max_batch = max_batch;
        pp->max_blocks = max_blocks_per_seq;
        pp->table.assign((size_t)max_batch * max_blocks_per_seq, -1);
        pp->lens.assign(max_batch, 0);
        pp->active.assign(max_batch, 0);
        pp->npages.assign(max_batch, 0);
        pp->ref.assign(num_pages, 0);
        pp->free_stack.resize(num_pages);
        pp->log.reserve(3 * (size_t)num_pages + 3 * 1024);
        pp->seen.assign((size_t)max_batch * max_blocks_per_seq, 0);
    } catch (...) {
        delete pp;
        return PKV_ERR_OOM;
    }
    // page 0 on top: a fresh pool hands pages out in increasing order
    for (int i = 0; i < num_pages; ++i) pp->free_stack[i] = num_pages - 1 - i;
    pp->free_top = num_pages;
    *out = pp;
    return PKV_OK;
}

pkv_status pkv_pages_destroy(pkv_pages* pp)
{
    delete pp;
    return PKV_OK;
}

pkv_status pkv_pages_admit(pkv_pages* pp, int slot, int len, int share_slot, int share_tokens)
{
    if (!slot_ok(pp, slot) || pp->active[slot] || len < 0) return PKV_ERR_INVALID_ARG;
    const int need = pages_for(len, pp->P);
    if (need > pp->max_blocks) return PKV_ERR_INVALID_ARG;
    int shared = 0;
    if (share_slot >= 0) {
        if (!slot_ok(pp, share_slot) || share_slot == slot || !pp->active[share_slot]) return PKV_ERR_INVALID_ARG;
        if (share_tokens < 0 || share_tokens > len || share_tokens > pp->lens[share_slot]) return PKV_ERR_INVALID_ARG;
        shared = share_tokens / pp->P;   // full pages only
    }
    if (need - shared > pp->free_top) return PKV_ERR_OOM;

    const int32_t* src = share_slot >= 0 ? &pp->table[(size_t)share_slot * pp->max_blocks] : nullptr;
    for (int i = 0; i < shared; ++i) {
        set_entry(pp, slot, i, src[i]);
        ++pp->ref[src[i]];
    }
    for (int i = shared; i < need; ++i) set_entry(pp, slot, i, pop_page(pp));
    pp->npages[slot] = need;
    pp->lens[slot] = len;
    pp->active[slot] = 1;
    return PKV_OK;
}

pkv_status pkv_pages_reserve(pkv_pages* pp, int q_len)
{
    if (!pp || q_len < 1) return PKV_ERR_INVALID_ARG;
    long long want = 0;
    for (int s = 0; s < pp->max_batch; ++s) {
        if (!pp->active[s]) continue;
        const int need = pages_for((long long)pp->lens[s] + q_len, pp->P);
        if (need > pp->max_blocks) return PKV_ERR_INVALID_ARG;
        if (need > pp->npages[s]) want += need - pp->npages[s];
    }
    if (want > pp->free_top) return PKV_ERR_OOM;
    for (int s = 0; s < pp->max_batch; ++s) {
        if (!pp->active[s]) continue;
        const int need = pages_for((long long)pp->lens[s] + q_len, pp->P);
        while (pp->npages[s] < need) {
            set_entry(pp, s, pp->npages[s], pop_page(pp));
            ++pp->npages[s];
        }
    }
    return PKV_OK;
}

pkv_status pkv_pages_advance(pkv_pages* pp, int q_len)
{
    if (!pp || q_len < 1) return PKV_ERR_INVALID_ARG;
    for (int s = 0; s < pp->max_batch; ++s)   // every active slot must hold pages for its new tokens
        if (pp->active[s] && pages_for((long long)pp->lens[s] + q_len, pp->P) > pp->npages[s])
            return PKV_ERR_INVALID_ARG;
    for (int s = 0; s < pp->max_batch; ++s)
        if (pp->active[s]) pp->lens[s] += q_len;
    return PKV_OK;
}

pkv_status pkv_pages_release(pkv_pages* pp, int slot)
{
    if (!slot_ok(pp, slot) || !pp->active[slot]) return PKV_ERR_INVALID_ARG;
    const int32_t* row = &pp->table[(size_t)slot * pp->max_blocks];
    for (int i = 0; i < pp->npages[slot]; ++i) {
        drop_page(pp, row[i]);
        set_entry(pp, slot, i, -1);
    }
    pp->npages[slot] = 0;
    pp->lens[slot] = 0;
    pp->active[slot] = 0;
    return PKV_OK;
}

const int32_t* pkv_pages_block_table(const pkv_pages* pp) { return pp ? pp->table.data() : nullptr; }
const int32_t* pkv_pages_seq_lens(const pkv_pages* pp) { return pp ? pp->lens.data() : nullptr; }
const int32_t* pkv_pages_active(const pkv_pages* pp) { return pp ? pp->active.data() : nullptr; }
const int32_t* pkv_pages_refcount(const pkv_pages* pp) { return pp ? pp->ref.data() : nullptr; }
int pkv_pages_free_count(const pkv_pages* pp) { return pp ? pp->free_top : -1; }

int pkv_pages_take_changes(pkv_pages* pp, int32_t* out, int max_changes)
{
    if (!pp || max_changes < 0 || (!out && max_changes > 0)) return -1;
    const int n = (int)(pp->log.size() / 3);
    int ret = -1;
    if (!pp->log_full) {
        // the last write of each entry, once, in the order of those writes:
        // walk the log backwards keeping first sightings, then reverse them
        const int32_t* lg = pp->log.data();
        int m = 0;
        bool fits = true;
        for (int k = n - 1; k >= 0; --k) {
            const size_t key = (size_t)lg[3 * k] * pp->max_blocks + lg[3 * k + 1];
            if (pp->seen[key]) continue;
            pp->seen[key] = 1;
            if (m >= max_changes) {
                fits = false;
                continue;   // keep marking, so the clean-up below finds every entry
            }
            out[3 * m] = lg[3 * k];
            out[3 * m + 1] = lg[3 * k + 1];
            out[3 * m + 2] = lg[3 * k + 2];
            ++m;
        }
        for (int k = 0; k < n; ++k) pp->seen[(size_t)lg[3 * k] * pp->max_blocks + lg[3 * k + 1]] = 0;
        if (fits) {
            for (int a = 0, b = m - 1; a < b; ++a, --b)
                for (int c = 0; c < 3; ++c) std::swap(out[3 * a + c], out[3 * b + c]);
            ret = m;
        }
    }
    pp->log.clear();
    pp->log_full = false;
    return ret;
}

}  // extern "C"
