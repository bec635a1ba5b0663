// Host block manager: the KV-cache manager of "Efficient Memory Management
// for Large Language Model Serving with PagedAttention" (summary page,
// section 2: logical-to-physical block mapping, on-demand allocation and
// reclamation, all-or-nothing eviction) with the sharing of section 1
// (reference counts plus copy-on-write for parallel samples and shared
// prefixes), over the global page pool of the "PyTorch-CUDA-v2.9 image
// enables PagedAttention" workflow list.  Host memory only.
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

struct pkv_block_manager {
    int num_blocks = 0;
    int block_size = 0;
    std::deque<int32_t> free_list;     // FIFO: head is handed out next
    std::vector<int32_t> ref;          // reference count per physical block
    std::vector<int32_t> fill;         // written token slots per physical block
    struct Seq {
        std::vector<int32_t> table;
        int64_t len = 0;
    };
    std::unordered_map<int64_t, Seq> seqs;
    int64_t used_blocks = 0;           // blocks with ref > 0

    int32_t take() {
        const int32_t b = free_list.front();
        free_list.pop_front();
        ref[b] = 1;
        fill[b] = 0;
        ++used_blocks;
        return b;
    }
    void release(int32_t b) {
        if (--ref[b] == 0) {
            fill[b] = 0;
            free_list.push_back(b);
            --used_blocks;
        }
    }
};

extern "C" {

pkv_status pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order,
                         pkv_block_manager** out) {
    if (!out || num_blocks <= 0 || block_size <= 0) return PKV_ERR_INVALID_ARG;
    pkv_block_manager* bm = new (std::nothrow) pkv_block_manager;
    if (!bm) return PKV_ERR_INVALID_ARG;
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->ref.assign(num_blocks, 0);
    bm->fill.assign(num_blocks, 0);
    if (free_order) {
        std::vector<char> seen(num_blocks, 0);
        for (int i = 0; i < num_blocks; ++i) {
            const int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete bm;
                return PKV_ERR_INVALID_ARG;
            }
            seen[b] = 1;
            bm->free_list.push_back(b);
        }
    } else {
        for (int i = 0; i < num_blocks; ++i) bm->free_list.push_back(i);
    }
    *out = bm;
    return PKV_OK;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

pkv_status pkv_bm_allocate(pkv_block_manager* bm, int64_t seq_id, int num_tokens) {
    if (!bm || num_tokens < 0) return PKV_ERR_INVALID_ARG;
    if (bm->seqs.count(seq_id)) return PKV_ERR_NOT_FOUND;
    const int64_t need = (num_tokens + (int64_t)bm->block_size - 1) / bm->block_size;
    if (need > (int64_t)bm->free_list.size()) return PKV_ERR_OUT_OF_BLOCKS;
    pkv_block_manager::Seq s;
    s.table.reserve(need);
    for (int64_t j = 0; j < need; ++j) {
        const int32_t b = bm->take();
        const int64_t left = num_tokens - j * bm->block_size;
        bm->fill[b] = (int32_t)(left < bm->block_size ? left : bm->block_size);
        s.table.push_back(b);
    }
    s.len = num_tokens;
    bm->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child) {
    if (!bm) return PKV_ERR_INVALID_ARG;
    auto it = bm->seqs.find(parent);
    if (it == bm->seqs.end() || bm->seqs.count(child)) return PKV_ERR_NOT_FOUND;
    pkv_block_manager::Seq s = it->second;
    for (int32_t b : s.table) ++bm->ref[b];
    bm->seqs.emplace(child, std::move(s));
    return PKV_OK;
}

pkv_status pkv_bm_append_slot(pkv_block_manager* bm, int64_t seq_id, int64_t* slot,
                              int32_t* cow_src, int32_t* cow_dst) {
    if (!bm || !slot || !cow_src || !cow_dst) return PKV_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PKV_ERR_NOT_FOUND;
    pkv_block_manager::Seq& s = it->second;
    const int64_t off = s.len % bm->block_size;
    int32_t src = -1, dst = -1;
    int32_t b;
    if (off == 0) {                         // last block full (or none): open a new one
        if (bm->free_list.empty()) return PKV_ERR_OUT_OF_BLOCKS;
        b = bm->take();
        s.table.push_back(b);
    } else {
        b = s.table.back();
        if (bm->ref[b] > 1) {               // shared, partly filled: copy on write
            if (bm->free_list.empty()) return PKV_ERR_OUT_OF_BLOCKS;
            const int32_t nb = bm->take();
            bm->fill[nb] = bm->fill[b];
            bm->release(b);
            s.table.back() = nb;
            src = b;
            dst = nb;
            b = nb;
        }
    }
    if (bm->fill[b] < off + 1) bm->fill[b] = (int32_t)(off + 1);
    ++s.len;
    *slot = (int64_t)b * bm->block_size + off;
    *cow_src = src;
    *cow_dst = dst;
    return PKV_OK;
}

pkv_status pkv_bm_append_slots(pkv_block_manager* bm, const int64_t* seq_ids, int n,
                               int64_t* slots, int64_t* cow_pairs, int* num_cow, int* num_done) {
    if (!bm || n < 0 || (n > 0 && (!seq_ids || !slots || !cow_pairs)) || !num_cow || !num_done)
        return PKV_ERR_INVALID_ARG;
    *num_cow = 0;
    *num_done = 0;
    for (int i = 0; i < n; ++i) {
        int32_t src, dst;
        const pkv_status st = pkv_bm_append_slot(bm, seq_ids[i], &slots[i], &src, &dst);
        if (st != PKV_OK) return st;
        if (src >= 0) {
            cow_pairs[2 * *num_cow] = src;
            cow_pairs[2 * *num_cow + 1] = dst;
            ++*num_cow;
        }
        ++*num_done;
    }
    return PKV_OK;
}

pkv_status pkv_bm_swap_out(pkv_block_manager* bm, pkv_block_manager* host, int64_t seq_id,
                           int64_t* pairs, int capacity, int* num_pairs) {
    if (!bm || !host || bm == host || !num_pairs || capacity < 0 || (capacity > 0 && !pairs))
        return PKV_ERR_INVALID_ARG;
    if (bm->block_size != host->block_size) return PKV_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || host->seqs.count(seq_id)) return PKV_ERR_NOT_FOUND;
    const std::vector<int32_t>& table = it->second.table;
    const int n = (int)table.size();
    *num_pairs = n;
    if (n > capacity) return PKV_ERR_INVALID_ARG;
    if ((size_t)n > host->free_list.size()) return PKV_ERR_OUT_OF_BLOCKS;   // nothing changed
    pkv_block_manager::Seq hs;
    hs.len = it->second.len;
    hs.table.reserve(n);
    for (int j = 0; j < n; ++j) {
        const int32_t d = host->take();
        host->fill[d] = bm->fill[table[j]];
        hs.table.push_back(d);
        pairs[2 * j] = table[j];
        pairs[2 * j + 1] = d;
    }
    host->seqs.emplace(seq_id, std::move(hs));
    for (int32_t b : table) bm->release(b);
    bm->seqs.erase(it);
    return PKV_OK;
}

pkv_status pkv_bm_free(pkv_block_manager* bm, int64_t seq_id) {
    if (!bm) return PKV_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PKV_ERR_NOT_FOUND;
    for (int32_t b : it->second.table) bm->release(b);
    bm->seqs.erase(it);
    return PKV_OK;
}

pkv_status pkv_bm_block_table(const pkv_block_manager* bm, int64_t seq_id, int32_t* out,
                              int capacity, int* num_blocks) {
    if (!bm || !num_blocks || capacity < 0 || (capacity > 0 && !out)) return PKV_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PKV_ERR_NOT_FOUND;
    const std::vector<int32_t>& t = it->second.table;
    *num_blocks = (int)t.size();
    for (int i = 0; i < capacity && i < (int)t.size(); ++i) out[i] = t[i];
    return PKV_OK;
}

pkv_status pkv_bm_fill_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int n,
                              int32_t* tables, int max_blocks_per_seq, int32_t* context_lens) {
    if (!bm || n < 0 || max_blocks_per_seq <= 0 || (n > 0 && (!seq_ids || !tables || !context_lens)))
        return PKV_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end()) return PKV_ERR_NOT_FOUND;
        const std::vector<int32_t>& t = it->second.table;
        if ((int)t.size() > max_blocks_per_seq) return PKV_ERR_INVALID_ARG;
        int32_t* row = tables + (size_t)i * max_blocks_per_seq;
        for (int j = 0; j < max_blocks_per_seq; ++j) row[j] = j < (int)t.size() ? t[j] : -1;
        context_lens[i] = (int32_t)it->second.len;
    }
    return PKV_OK;
}

int pkv_bm_num_free(const pkv_block_manager* bm) { return bm ? (int)bm->free_list.size() : -1; }

int pkv_bm_seq_len(const pkv_block_manager* bm, int64_t seq_id) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : (int)it->second.len;
}

int pkv_bm_ref_count(const pkv_block_manager* bm, int32_t block) {
    if (!bm || block < 0 || block >= bm->num_blocks) return -1;
    return bm->ref[block];
}

double pkv_bm_utilisation(const pkv_block_manager* bm) {
    if (!bm || bm->used_blocks == 0) return 0.0;
    int64_t filled = 0;
    for (int b = 0; b < bm->num_blocks; ++b)
        if (bm->ref[b] > 0) filled += bm->fill[b];
    return (double)filled / ((double)bm->used_blocks * bm->block_size);
}

}  // extern "C"
