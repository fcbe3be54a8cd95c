// moe_cache.cu -- expert cache: packed layers in host memory, the experts a call needs copied into
// a fixed pool of device slots, behind per-layer headers that the forward kernels read as packed
// layers (include/moe.h, "Expert cache").
//
// Host code only; the device sees the pool through ordinary copies on the caller's stream.
// Pool layout: [header of layer 0 .. layer L-1][slot 0 .. slot S-1]. Every header and slot starts
// on a 256-byte boundary, so every entry offset (slot address minus header address) is positive,
// a multiple of 256 and below 2^40, as the forward kernels require.
//
// Bookkeeping per request: slot_of[layer*E + e] (slot or -1), owner[slot] (layer*E + e or -1) and
// last_req[slot] (number of the last request that named the slot's expert). A request writes an
// undo log, so that a request replaced before its commit, or a commit whose copies fail, leaves
// the cache as if it had not happened (a failed commit frees the slots it was filling: their
// previous bytes may already be overwritten).
#include <algorithm>
#include <cstring>
#include <memory>
#include <new>
#include <vector>

#include "moe_internal.cuh"

using moe::PackedExpert;
using moe::PackedHeader;

struct moe_expert_cache {
    int L = 0, E = 0, H = 0, I = 0, slots = 0, keep_recent = 1;
    uint8_t *pool = nullptr;   // device
    size_t hdr_bytes = 0, slot_bytes = 0;
    std::vector<const uint8_t *> host;             // [L] packed layers in host memory
    std::vector<PackedExpert> src;                 // [L*E] their entries (offset within the host layer)
    std::vector<std::vector<uint8_t>> mirror;      // [L] host image of each device header
    std::vector<int32_t> slot_of;                  // [L*E]
    std::vector<int64_t> owner;                    // [slots]
    std::vector<uint64_t> last_req;                // [slots]
    uint64_t nreq = 0;
    uint64_t hits = 0, misses = 0, evictions = 0;

    struct Undo {
        int32_t slot;
        int64_t prev_owner;   // owner before the request (unchanged for a hit)
        uint64_t prev_last;
        bool load;            // a missing expert was given this slot
    };
    bool pending = false;
    int cur_layer = -1;
    std::vector<Undo> undo;
    uint64_t d_hits = 0, d_misses = 0, d_evictions = 0;

    size_t slot_base() const { return (size_t)L * hdr_bytes; }
    size_t slot_addr(int s) const { return slot_base() + (size_t)s * slot_bytes; }

    // puts back everything the pending request changed
    void rollback() {
        for (auto it = undo.rbegin(); it != undo.rend(); ++it) {
            if (it->load) {
                slot_of[(size_t)owner[it->slot]] = -1;
                if (it->prev_owner >= 0) slot_of[(size_t)it->prev_owner] = it->slot;
                owner[it->slot] = it->prev_owner;
            }
            last_req[it->slot] = it->prev_last;
        }
        hits -= d_hits;
        misses -= d_misses;
        evictions -= d_evictions;
        --nreq;
        undo.clear();
        pending = false;
        cur_layer = -1;
    }

    // after a failed commit: the slots being filled are freed (their old contents may be gone)
    void drop_loads() {
        for (const Undo &u : undo)
            if (u.load) {
                slot_of[(size_t)owner[u.slot]] = -1;
                owner[u.slot] = -1;
                last_req[u.slot] = 0;
            }
        undo.clear();
        pending = false;
        cur_layer = -1;
    }
};

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct LayerShape {
    int E = 0, H = 0, I = 0;
    size_t max_expert = 0;
};

// Reads and checks the packed headers of the host layers; false if any is malformed.
bool read_layers(int L, const void *const *host_layers, const size_t *host_bytes, LayerShape &shape,
                 std::vector<PackedExpert> *entries) {
    if (L < 1 || !host_layers || !host_bytes) return false;
    for (int l = 0; l < L; ++l) {
        const uint8_t *p = static_cast<const uint8_t *>(host_layers[l]);
        if (!p || host_bytes[l] < sizeof(PackedHeader)) return false;
        PackedHeader h;
        std::memcpy(&h, p, sizeof h);
        if (h.magic != moe::kPackedMagic || h.version != moe::kPackedVersion) return false;
        if (h.E < 1 || h.E > moe::kMaxE || h.H < 64 || h.H % moe::kGroup || h.I < 64 || h.I % moe::kGroup) return false;
        if (l == 0) {
            shape.E = h.E;
            shape.H = h.H;
            shape.I = h.I;
        } else if (h.E != shape.E || h.H != shape.H || h.I != shape.I) {
            return false;
        }
        const size_t start = moe::packed_data_start(h.E);
        if (host_bytes[l] < start) return false;
        for (int e = 0; e < h.E; ++e) {
            PackedExpert x;
            std::memcpy(&x, p + sizeof(PackedHeader) + (size_t)e * sizeof(PackedExpert), sizeof x);
            if (x.bits != 4 && x.bits != 6 && x.bits != 8) return false;
            const size_t nb = moe::expert_bytes(h.H, h.I, x.bits);
            if (x.offset < start || x.offset % 256 || x.offset > host_bytes[l] || host_bytes[l] - x.offset < nb)
                return false;
            shape.max_expert = std::max(shape.max_expert, nb);
            if (entries) entries->push_back(x);
        }
    }
    return true;
}

size_t pool_bytes_for(int L, const LayerShape &s, int slots, size_t *hdr, size_t *slot) {
    const size_t h = moe::packed_data_start(s.E);
    const size_t sb = moe::align_up(s.max_expert, 256);
    if (hdr) *hdr = h;
    if (slot) *slot = sb;
    return (size_t)L * h + (size_t)slots * sb;
}

constexpr size_t kMaxPool = (size_t)1 << 40;   // entry offsets are kept as offset / 256 in 32 bits

}  // namespace

extern "C" {

size_t moe_cache_pool_bytes(int L, const void *const *host_layers, const size_t *host_bytes, int slots) {
    LayerShape s;
    if (slots < 1 || !read_layers(L, host_layers, host_bytes, s, nullptr)) return 0;
    const size_t n = pool_bytes_for(L, s, slots, nullptr, nullptr);
    return n < kMaxPool ? n : 0;
}

moe_status_t moe_cache_create(int L, const void *const *host_layers, const size_t *host_bytes, int slots,
                              int keep_recent, void *pool, size_t pool_bytes, moe_expert_cache_t **cache) {
    if (!cache) return MOE_ERR_INVALID_ARG;
    *cache = nullptr;
    if (slots < 1 || keep_recent < 1 || keep_recent > 8 || !pool || !aligned(pool, 256)) return MOE_ERR_INVALID_ARG;
    try {
        LayerShape s;
        std::vector<PackedExpert> entries;
        if (!read_layers(L, host_layers, host_bytes, s, &entries)) return MOE_ERR_INVALID_ARG;
        size_t hdr = 0, sb = 0;
        const size_t need = pool_bytes_for(L, s, slots, &hdr, &sb);
        if (need >= kMaxPool || pool_bytes < need) return MOE_ERR_INVALID_ARG;
        std::unique_ptr<moe_expert_cache> c(new moe_expert_cache());
        c->L = L;
        c->E = s.E;
        c->H = s.H;
        c->I = s.I;
        c->slots = slots;
        c->keep_recent = keep_recent;
        c->pool = static_cast<uint8_t *>(pool);
        c->hdr_bytes = hdr;
        c->slot_bytes = sb;
        c->src = std::move(entries);
        c->slot_of.assign((size_t)L * s.E, -1);
        c->owner.assign(slots, -1);
        c->last_req.assign(slots, 0);
        c->host.resize(L);
        c->mirror.resize(L);
        for (int l = 0; l < L; ++l) {
            c->host[l] = static_cast<const uint8_t *>(host_layers[l]);
            // the device header starts with every entry on slot 0: in bounds, whatever it holds
            std::vector<uint8_t> &m = c->mirror[l];
            m.assign(hdr, 0);
            PackedHeader h = {};
            h.magic = moe::kPackedMagic;
            h.version = moe::kPackedVersion;
            h.E = s.E;
            h.H = s.H;
            h.I = s.I;
            std::memcpy(m.data(), &h, sizeof h);
            for (int e = 0; e < s.E; ++e) {
                PackedExpert x = {c->slot_addr(0) - (size_t)l * hdr, c->src[(size_t)l * s.E + e].bits, 0};
                std::memcpy(m.data() + sizeof(PackedHeader) + (size_t)e * sizeof(PackedExpert), &x, sizeof x);
            }
        }
        *cache = c.release();
        return MOE_OK;
    } catch (const std::bad_alloc &) {
        return MOE_ERR_UNSUPPORTED;   // host memory exhausted
    }
}

void moe_cache_destroy(moe_expert_cache_t *cache) { delete cache; }

moe_status_t moe_cache_request(moe_expert_cache_t *c, int layer, const int32_t *experts, int n,
                               int32_t *load_experts, int32_t *load_slots, int *n_load) {
    if (!c || !n_load || layer < 0 || layer >= c->L || n < 0 || (n > 0 && !experts)) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (experts[i] < 0 || experts[i] >= c->E) return MOE_ERR_INVALID_ARG;
    try {
        if (c->pending) c->rollback();
        const uint64_t req = c->nreq + 1;
        // distinct experts, first occurrence order
        std::vector<int32_t> want;
        std::vector<char> seen((size_t)c->E, 0);
        for (int i = 0; i < n; ++i)
            if (!seen[(size_t)experts[i]]) {
                seen[(size_t)experts[i]] = 1;
                want.push_back(experts[i]);
            }
        const size_t base = (size_t)layer * c->E;
        size_t nmiss = 0;
        for (int32_t e : want) nmiss += c->slot_of[base + (size_t)e] < 0;
        // slots a missing expert may take: free ones first, then the least recently requested
        // among those no recent request named (hits of this request are named by it)
        std::vector<int32_t> cand;
        for (int s = 0; s < c->slots; ++s)
            if (c->owner[s] < 0) cand.push_back(s);
        std::vector<int32_t> lru;
        for (int s = 0; s < c->slots; ++s) {
            if (c->owner[s] < 0) continue;
            const int64_t o = c->owner[s];
            const bool hit_now = o / c->E == layer && seen[(size_t)(o % c->E)];
            const bool recent = c->last_req[s] + (uint64_t)c->keep_recent > req;   // named by one of the last keep_recent - 1
            if (!hit_now && !recent) lru.push_back(s);
        }
        if (cand.size() + lru.size() < nmiss) return MOE_ERR_UNSUPPORTED;
        std::stable_sort(lru.begin(), lru.end(),
                         [c](int32_t a, int32_t b) { return c->last_req[a] < c->last_req[b]; });
        cand.insert(cand.end(), lru.begin(), lru.end());

        c->nreq = req;
        c->undo.clear();
        c->d_hits = c->d_misses = c->d_evictions = 0;
        size_t next = 0;
        int nl = 0;
        for (int32_t e : want) {
            const size_t key = base + (size_t)e;
            int32_t s = c->slot_of[key];
            if (s >= 0) {
                c->undo.push_back({s, c->owner[s], c->last_req[s], false});
                c->last_req[s] = req;
                ++c->d_hits;
                continue;
            }
            s = cand[next++];
            const int64_t prev = c->owner[s];
            c->undo.push_back({s, prev, c->last_req[s], true});
            if (prev >= 0) {
                c->slot_of[(size_t)prev] = -1;
                ++c->d_evictions;
            }
            c->owner[s] = (int64_t)key;
            c->slot_of[key] = s;
            c->last_req[s] = req;
            ++c->d_misses;
            if (load_experts) load_experts[nl] = e;
            if (load_slots) load_slots[nl] = s;
            ++nl;
        }
        c->hits += c->d_hits;
        c->misses += c->d_misses;
        c->evictions += c->d_evictions;
        c->pending = true;
        c->cur_layer = layer;
        *n_load = nl;
        return MOE_OK;
    } catch (const std::bad_alloc &) {
        return MOE_ERR_UNSUPPORTED;
    }
}

moe_status_t moe_cache_commit(moe_expert_cache_t *c, moe_stream_t stream, const void **packed) {
    if (!c || !packed || !c->pending) return MOE_ERR_INVALID_ARG;
    const moe_status_t dev = moe::require_sm100();
    if (dev != MOE_OK) {
        c->rollback();
        return dev;
    }
    const int l = c->cur_layer;
    const cudaStream_t st = (cudaStream_t)stream;
    std::vector<uint8_t> &m = c->mirror[l];
    for (const auto &u : c->undo) {
        if (!u.load) continue;
        const int e = (int)(c->owner[u.slot] % c->E);
        const PackedExpert &x = c->src[(size_t)l * c->E + e];
        const size_t nb = moe::expert_bytes(c->H, c->I, x.bits);
        if (cudaMemcpyAsync(c->pool + c->slot_addr(u.slot), c->host[l] + x.offset, nb, cudaMemcpyHostToDevice,
                            st) != cudaSuccess) {
            c->drop_loads();
            return MOE_ERR_CUDA;
        }
        const PackedExpert y = {c->slot_addr(u.slot) - (size_t)l * c->hdr_bytes, x.bits, 0};
        std::memcpy(m.data() + sizeof(PackedHeader) + (size_t)e * sizeof(PackedExpert), &y, sizeof y);
    }
    uint8_t *hdr = c->pool + (size_t)l * c->hdr_bytes;
    if (cudaMemcpyAsync(hdr, m.data(), c->hdr_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) {
        c->drop_loads();
        return MOE_ERR_CUDA;
    }
    c->undo.clear();
    c->pending = false;
    c->cur_layer = -1;
    *packed = hdr;
    return MOE_OK;
}

int moe_cache_slot_of(const moe_expert_cache_t *c, int layer, int expert) {
    if (!c || layer < 0 || layer >= c->L || expert < 0 || expert >= c->E) return -1;
    return c->slot_of[(size_t)layer * c->E + expert];
}

moe_status_t moe_cache_stats(const moe_expert_cache_t *c, uint64_t *hits, uint64_t *misses, uint64_t *evictions) {
    if (!c) return MOE_ERR_INVALID_ARG;
    if (hits) *hits = c->hits;
    if (misses) *misses = c->misses;
    if (evictions) *evictions = c->evictions;
    return MOE_OK;
}

}  // extern "C"
