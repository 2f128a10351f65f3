// Host-side block manager for the paged KV pool, plus the device page copy
// that copy-on-write needs.
//
// The pages' allocator semantics: GPU memory cut into fixed-size blocks handed
// out on demand and released atomically ("大模型推理优化：KV Cache与FlashAttention
// 实战" §4.1, 块级内存池); identical prompts share KV blocks, with reference
// counts managing their lifetime (§4.1 零拷贝共享; "LLM推理系统优化：KV缓存管理与
// 动态批处理技术" §3.1, shared system-prompt blocks); a page table maps each
// sequence's logical pages to physical ones ("Flash Attention与Paged KV Cache
// 优化大模型计算效率" §3.2), and releasing a sequence must delete its page-table
// entries, the fix of the leak described in that page's §5.2.
//
// Model: a sequence is a list of physical pages plus a token count.  fork()
// gives the child the parent's pages (every refcount + 1).  append() reserves
// slots for new tokens at the end of a sequence: when the last page is shared
// and has room, it is first replaced by a private copy (copy-on-write; the
// caller copies the page on the device with pkv_copy_pages before writing new
// rows), then new pages are taken from the free list as needed.  free()
// drops the sequence's references and deletes its entry; pages whose count
// reaches zero return to the free list.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "pkv_kernels.h"

struct pkv_block_manager {
    std::mutex mu;
    int64_t num_pages;
    int page_size;
    int max_pages_per_seq;
    std::vector<int32_t> refcount;      // per physical page
    std::vector<int32_t> free_list;     // LIFO of free pages
    struct Seq {
        std::vector<int32_t> pages;
        int64_t tokens = 0;
    };
    std::unordered_map<int64_t, Seq> seqs;
    int64_t next_id = 0;

    int32_t take_page() {
        const int32_t p = free_list.back();
        free_list.pop_back();
        refcount[p] = 1;
        return p;
    }
    void drop_page(int32_t p) {
        if (--refcount[p] == 0) free_list.push_back(p);
    }
};

namespace {

// Copy whole pages (page_bytes each) src[i] -> dst[i] of the K and V pools;
// one CTA per page pair, 16-byte vectors when the sizes allow.
template <typename V>
__global__ void __launch_bounds__(256)
copy_pages_kernel(uint8_t* __restrict__ kp, uint8_t* __restrict__ vp, const int32_t* __restrict__ src,
                  const int32_t* __restrict__ dst, int64_t page_bytes, int64_t num_pages, pkv::DeviceStatus* status) {
    const int i = blockIdx.x;
    const int32_t s = __ldg(src + i), d = __ldg(dst + i);
    if (s < 0 || d < 0 || s >= num_pages || d >= num_pages) {
        if (threadIdx.x == 0) pkv::record_error(status, PKV_ERR_DEVICE_RANGE, s < 0 || s >= num_pages ? s : d);
        return;
    }
    const int64_t n = page_bytes / static_cast<int64_t>(sizeof(V));
    const V* ks = reinterpret_cast<const V*>(kp + s * page_bytes);
    const V* vs = reinterpret_cast<const V*>(vp + s * page_bytes);
    V* kd = reinterpret_cast<V*>(kp + d * page_bytes);
    V* vd = reinterpret_cast<V*>(vp + d * page_bytes);
    for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
        const V a = ks[j], b = vs[j];
        kd[j] = a;
        vd[j] = b;
    }
}

}  // namespace

namespace pkv {
DeviceStatus* device_status_ptr();   // api.cu
}

extern "C" {

pkv_block_manager* pkv_bm_create(int64_t num_pages, int page_size, int max_pages_per_seq) {
    if (num_pages <= 0 || num_pages > INT32_MAX || page_size <= 0 || max_pages_per_seq <= 0) return nullptr;
    auto* bm = new (std::nothrow) pkv_block_manager();
    if (!bm) return nullptr;
    bm->num_pages = num_pages;
    bm->page_size = page_size;
    bm->max_pages_per_seq = max_pages_per_seq;
    bm->refcount.assign(static_cast<size_t>(num_pages), 0);
    bm->free_list.reserve(static_cast<size_t>(num_pages));
    for (int64_t p = num_pages - 1; p >= 0; --p) bm->free_list.push_back(static_cast<int32_t>(p));
    return bm;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

int pkv_bm_add_sequence(pkv_block_manager* bm, int64_t* seq_id_out) {
    if (!bm || !seq_id_out) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(bm->mu);
    const int64_t id = bm->next_id++;
    bm->seqs.emplace(id, pkv_block_manager::Seq{});
    *seq_id_out = id;
    return PKV_OK;
}

int pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t* child_out) {
    if (!bm || !child_out) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(bm->mu);
    auto it = bm->seqs.find(parent);
    if (it == bm->seqs.end()) return PKV_ERR_INVALID_ARG;
    pkv_block_manager::Seq child = it->second;
    for (int32_t p : child.pages) ++bm->refcount[p];
    const int64_t id = bm->next_id++;
    bm->seqs.emplace(id, std::move(child));
    *child_out = id;
    return PKV_OK;
}

int pkv_bm_append(pkv_block_manager* bm, int64_t seq, int num_tokens, int64_t* slots_out, int32_t* copy_src,
                  int32_t* copy_dst, int* num_copies) {
    if (!bm || num_tokens < 0 || (num_tokens > 0 && !slots_out) || !num_copies) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(bm->mu);
    *num_copies = 0;
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end()) return PKV_ERR_INVALID_ARG;
    auto& s = it->second;
    const int ps = bm->page_size;
    const int64_t total = s.tokens + num_tokens;
    const int64_t need_pages = (total + ps - 1) / ps;
    if (need_pages > bm->max_pages_per_seq) return PKV_ERR_INVALID_ARG;
    const bool cow = num_tokens > 0 && (s.tokens % ps) != 0 && bm->refcount[s.pages.back()] > 1;
    const int64_t new_pages = need_pages - static_cast<int64_t>(s.pages.size()) + (cow ? 1 : 0);
    if (new_pages > static_cast<int64_t>(bm->free_list.size())) return PKV_ERR_OUT_OF_PAGES;
    if (cow) {
        if (!copy_src || !copy_dst) return PKV_ERR_INVALID_ARG;
        const int32_t old = s.pages.back();
        const int32_t fresh = bm->take_page();
        bm->drop_page(old);
        s.pages.back() = fresh;
        copy_src[0] = old;
        copy_dst[0] = fresh;
        *num_copies = 1;
    }
    while (static_cast<int64_t>(s.pages.size()) < need_pages) s.pages.push_back(bm->take_page());
    for (int i = 0; i < num_tokens; ++i) {
        const int64_t pos = s.tokens + i;
        slots_out[i] = static_cast<int64_t>(s.pages[static_cast<size_t>(pos / ps)]) * ps + pos % ps;
    }
    s.tokens = total;
    return PKV_OK;
}

int pkv_bm_free_sequence(pkv_block_manager* bm, int64_t seq) {
    if (!bm) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(bm->mu);
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end()) return PKV_ERR_INVALID_ARG;     // unknown or already freed
    for (int32_t p : it->second.pages) bm->drop_page(p);
    bm->seqs.erase(it);                                        // the table entry goes too
    return PKV_OK;
}

int pkv_bm_block_tables(pkv_block_manager* bm, const int64_t* seq_ids, int num_seqs, int32_t* table_out,
                        int32_t* context_lens_out) {
    if (!bm || num_seqs < 0 || (num_seqs > 0 && (!seq_ids || !table_out || !context_lens_out)))
        return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(bm->mu);
    const int mp = bm->max_pages_per_seq;
    for (int b = 0; b < num_seqs; ++b) {
        auto it = bm->seqs.find(seq_ids[b]);
        if (it == bm->seqs.end()) return PKV_ERR_INVALID_ARG;
        const auto& pages = it->second.pages;
        for (int j = 0; j < mp; ++j)
            table_out[static_cast<int64_t>(b) * mp + j] = j < static_cast<int>(pages.size()) ? pages[j] : -1;
        context_lens_out[b] = static_cast<int32_t>(it->second.tokens);
    }
    return PKV_OK;
}

int64_t pkv_bm_num_free_pages(pkv_block_manager* bm) {
    if (!bm) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(bm->mu);
    return static_cast<int64_t>(bm->free_list.size());
}

int pkv_bm_page_refcount(pkv_block_manager* bm, int32_t page) {
    if (!bm) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(bm->mu);
    if (page < 0 || page >= bm->num_pages) return PKV_ERR_INVALID_ARG;
    return bm->refcount[page];
}

int pkv_bm_num_sequences(pkv_block_manager* bm) {
    if (!bm) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(bm->mu);
    return static_cast<int>(bm->seqs.size());
}

int pkv_copy_pages(void* k_pages, void* v_pages, const int32_t* src, const int32_t* dst, int num_copies,
                   int64_t page_bytes, int64_t num_pages, pkv_stream_t stream) {
    if (num_copies < 0 || page_bytes <= 0 || num_pages <= 0) return PKV_ERR_INVALID_ARG;
    if (num_copies == 0) return PKV_OK;
    if (!k_pages || !v_pages || !src || !dst) return PKV_ERR_INVALID_ARG;
    pkv::DeviceStatus* st = pkv::device_status_ptr();
    if (!st) return PKV_ERR_CUDA;
    auto s = reinterpret_cast<cudaStream_t>(stream);
    auto* kp = static_cast<uint8_t*>(k_pages);
    auto* vp = static_cast<uint8_t*>(v_pages);
    const uintptr_t align = reinterpret_cast<uintptr_t>(kp) | reinterpret_cast<uintptr_t>(vp) |
                            static_cast<uintptr_t>(page_bytes);
    if (align % 16 == 0)
        copy_pages_kernel<uint4><<<num_copies, 256, 0, s>>>(kp, vp, src, dst, page_bytes, num_pages, st);
    else
        copy_pages_kernel<uint8_t><<<num_copies, 256, 0, s>>>(kp, vp, src, dst, page_bytes, num_pages, st);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // extern "C"
