// Block manager and block-copy kernel of libpagedattn.
//
// The manager produces the block tables pa_decode consumes.  It follows the
// PagedAttention idea as the pages state it ("vLLM 0.25.0 release-notes
// commentary", section 1; "Why PagedAttention was retired", section 1): a
// sequence is like a process, a KV block like a page and the block table like
// a page table; blocks are allocated only when a sequence needs them, and
// several outputs can share one prompt's blocks, copying a shared block on
// write.  The host side is plain C++ (one mutex per manager); the copies a
// copy-on-write needs run on the GPU in pa_copy_blocks_kernel.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "pagedattn.h"

namespace {

thread_local char g_bm_detail[256] = "";

pa_status bm_fail(pa_status st, const char* what) {
    std::snprintf(g_bm_detail, sizeof g_bm_detail, "%s", what);
    return st;
}

}  // namespace

struct pa_block_manager {
    struct Seq {
        bool live = false;
        int64_t len = 0;
        std::vector<int32_t> blocks;
    };
    int64_t num_blocks = 0;
    int block_size = 0;
    int max_blocks_per_seq = 0;
    std::vector<int32_t> refcount;  // per physical block
    std::vector<int32_t> free_ids;  // stack; the next allocation pops the back
    std::vector<Seq> seqs;          // indexed by sequence id
    std::vector<int> free_seq_ids;
    std::mutex mu;

    int32_t pop_block() {
        const int32_t b = free_ids.back();
        free_ids.pop_back();
        refcount[b] = 1;
        return b;
    }
    void release(int32_t b) {
        if (--refcount[b] == 0) free_ids.push_back(b);
    }
    bool valid_seq(int id) const {
        return id >= 0 && id < static_cast<int>(seqs.size()) && seqs[id].live;
    }
    int new_seq_id() {
        if (!free_seq_ids.empty()) {
            const int id = free_seq_ids.back();
            free_seq_ids.pop_back();
            return id;
        }
        seqs.emplace_back();
        return static_cast<int>(seqs.size()) - 1;
    }
};

extern "C" {

pa_status pa_bm_create(pa_block_manager** out, int64_t num_blocks, int block_size,
                       int max_blocks_per_seq) {
    g_bm_detail[0] = 0;
    if (!out) return bm_fail(PA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (num_blocks < 1 || num_blocks > 0x7fffffffLL)
        return bm_fail(PA_ERR_INVALID_ARG, "num_blocks must be in [1, 2^31)");
    if (block_size < 1) return bm_fail(PA_ERR_INVALID_ARG, "block_size < 1");
    if (max_blocks_per_seq < 1) return bm_fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq < 1");
    pa_block_manager* m = new (std::nothrow) pa_block_manager();
    if (!m) return bm_fail(PA_ERR_INVALID_ARG, "out of host memory");
    m->num_blocks = num_blocks;
    m->block_size = block_size;
    m->max_blocks_per_seq = max_blocks_per_seq;
    m->refcount.assign(static_cast<size_t>(num_blocks), 0);
    m->free_ids.resize(static_cast<size_t>(num_blocks));
    // Highest id at the bottom of the stack: allocation hands out 0, 1, 2, ...
    for (int64_t i = 0; i < num_blocks; ++i)
        m->free_ids[static_cast<size_t>(i)] = static_cast<int32_t>(num_blocks - 1 - i);
    *out = m;
    return PA_OK;
}

void pa_bm_destroy(pa_block_manager* m) { delete m; }

pa_status pa_bm_add_sequence(pa_block_manager* m, int* seq_id) {
    g_bm_detail[0] = 0;
    if (!m || !seq_id) return bm_fail(PA_ERR_INVALID_ARG, "NULL argument");
    std::lock_guard<std::mutex> g(m->mu);
    const int id = m->new_seq_id();
    m->seqs[id].live = true;
    m->seqs[id].len = 0;
    m->seqs[id].blocks.clear();
    *seq_id = id;
    return PA_OK;
}

pa_status pa_bm_fork(pa_block_manager* m, int parent, int* child) {
    g_bm_detail[0] = 0;
    if (!m || !child) return bm_fail(PA_ERR_INVALID_ARG, "NULL argument");
    std::lock_guard<std::mutex> g(m->mu);
    if (!m->valid_seq(parent)) return bm_fail(PA_ERR_INVALID_ARG, "parent is not a live sequence");
    const int id = m->new_seq_id();  // may grow seqs: take the parent by index after
    pa_block_manager::Seq& c = m->seqs[id];
    const pa_block_manager::Seq& p = m->seqs[parent];
    c.live = true;
    c.len = p.len;
    c.blocks = p.blocks;
    for (int32_t b : c.blocks) ++m->refcount[b];
    *child = id;
    return PA_OK;
}

pa_status pa_bm_free_sequence(pa_block_manager* m, int seq) {
    g_bm_detail[0] = 0;
    if (!m) return bm_fail(PA_ERR_INVALID_ARG, "NULL manager");
    std::lock_guard<std::mutex> g(m->mu);
    if (!m->valid_seq(seq)) return bm_fail(PA_ERR_INVALID_ARG, "not a live sequence");
    pa_block_manager::Seq& s = m->seqs[seq];
    for (int32_t b : s.blocks) m->release(b);
    s.blocks.clear();
    s.len = 0;
    s.live = false;
    m->free_seq_ids.push_back(seq);
    return PA_OK;
}

pa_status pa_bm_append_tokens(pa_block_manager* m, int seq, int num_tokens, int64_t* copy_src,
                              int64_t* copy_dst, int* num_copies) {
    g_bm_detail[0] = 0;
    if (!m || !num_copies) return bm_fail(PA_ERR_INVALID_ARG, "NULL argument");
    *num_copies = 0;
    if (num_tokens < 0) return bm_fail(PA_ERR_INVALID_ARG, "num_tokens < 0");
    std::lock_guard<std::mutex> g(m->mu);
    if (!m->valid_seq(seq)) return bm_fail(PA_ERR_INVALID_ARG, "not a live sequence");
    pa_block_manager::Seq& s = m->seqs[seq];
    if (num_tokens == 0) return PA_OK;
    const int64_t B = m->block_size;
    const int64_t new_len = s.len + num_tokens;
    const int64_t need = (new_len + B - 1) / B;
    const int64_t have = static_cast<int64_t>(s.blocks.size());
    if (need > m->max_blocks_per_seq)
        return bm_fail(PA_ERR_OUT_OF_BLOCKS, "sequence would exceed max_blocks_per_seq");
    // Writing into a partly filled last block that another sequence also maps
    // needs a private copy first (copy on write).
    const bool cow = (s.len % B) != 0 && have > 0 && m->refcount[s.blocks.back()] > 1;
    const int64_t fresh = (need - have) + (cow ? 1 : 0);
    if (fresh > static_cast<int64_t>(m->free_ids.size()))
        return bm_fail(PA_ERR_OUT_OF_BLOCKS, "not enough free blocks");
    if (cow && (!copy_src || !copy_dst))
        return bm_fail(PA_ERR_INVALID_ARG, "a copy on write is needed: copy_src/copy_dst are NULL");
    if (cow) {
        const int32_t old = s.blocks.back();
        const int32_t nb = m->pop_block();
        m->release(old);
        s.blocks.back() = nb;
        *copy_src = old;
        *copy_dst = nb;
        *num_copies = 1;
    }
    for (int64_t i = have; i < need; ++i) s.blocks.push_back(m->pop_block());
    s.len = new_len;
    return PA_OK;
}

pa_status pa_bm_seq_len(pa_block_manager* m, int seq, int64_t* len) {
    g_bm_detail[0] = 0;
    if (!m || !len) return bm_fail(PA_ERR_INVALID_ARG, "NULL argument");
    std::lock_guard<std::mutex> g(m->mu);
    if (!m->valid_seq(seq)) return bm_fail(PA_ERR_INVALID_ARG, "not a live sequence");
    *len = m->seqs[seq].len;
    return PA_OK;
}

pa_status pa_bm_export(pa_block_manager* m, const int* seq_ids, int n, int32_t* block_tables,
                       int max_blocks_per_seq, int32_t* seq_lens) {
    g_bm_detail[0] = 0;
    if (!m || (n > 0 && (!seq_ids || !block_tables || !seq_lens)))
        return bm_fail(PA_ERR_INVALID_ARG, "NULL argument");
    if (n < 0) return bm_fail(PA_ERR_INVALID_ARG, "n < 0");
    std::lock_guard<std::mutex> g(m->mu);
    for (int i = 0; i < n; ++i) {
        if (!m->valid_seq(seq_ids[i])) return bm_fail(PA_ERR_INVALID_ARG, "not a live sequence");
        if (static_cast<int64_t>(m->seqs[seq_ids[i]].blocks.size()) > max_blocks_per_seq)
            return bm_fail(PA_ERR_INVALID_ARG, "a sequence has more blocks than the row holds");
        if (m->seqs[seq_ids[i]].len > 0x7fffffffLL)
            return bm_fail(PA_ERR_INVALID_ARG, "sequence longer than int32");
    }
    for (int i = 0; i < n; ++i) {
        const pa_block_manager::Seq& s = m->seqs[seq_ids[i]];
        int32_t* row = block_tables + static_cast<int64_t>(i) * max_blocks_per_seq;
        const size_t nb = s.blocks.size();
        if (nb) std::memcpy(row, s.blocks.data(), nb * sizeof(int32_t));
        for (int j = static_cast<int>(nb); j < max_blocks_per_seq; ++j) row[j] = -1;
        seq_lens[i] = static_cast<int32_t>(s.len);
    }
    return PA_OK;
}

int64_t pa_bm_num_free_blocks(pa_block_manager* m) {
    if (!m) return -1;
    std::lock_guard<std::mutex> g(m->mu);
    return static_cast<int64_t>(m->free_ids.size());
}

int pa_bm_refcount(pa_block_manager* m, int64_t block) {
    if (!m || block < 0 || block >= m->num_blocks) return -1;
    std::lock_guard<std::mutex> g(m->mu);
    return m->refcount[static_cast<size_t>(block)];
}

const char* pa_bm_last_error_detail(void) { return g_bm_detail; }

}  // extern "C"

// ------------------------------------------------------------ block copies
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

// One CTA per (pair, cache half, slice): copies `slice` 16-byte words of one
// block's K (blockIdx.y == 0) or V (== 1) bytes from block src[i] to dst[i].
// Pairs with an id outside [0, num_blocks) are skipped and flagged.
__global__ void __launch_bounds__(kCopyThreads) pa_copy_blocks_kernel(
    uint8_t* key_cache, uint8_t* value_cache, long long block_words, long long slice_words,
    const int64_t* src, const int64_t* dst, long long num_blocks, uint32_t* status) {
    const long long i = blockIdx.x;
    const int64_t a = src[i];
    const int64_t b = dst[i];
    if (a < 0 || a >= num_blocks || b < 0 || b >= num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && status)
            atomicOr(status, PA_DEV_BAD_BLOCK_ID);
        return;
    }
    uint8_t* base = blockIdx.y == 0 ? key_cache : value_cache;
    const uint4* from = reinterpret_cast<const uint4*>(base) + a * block_words;
    uint4* to = reinterpret_cast<uint4*>(base) + b * block_words;
    const long long w0 = blockIdx.z * slice_words;
    const long long w1 = min(block_words, w0 + slice_words);
    for (long long w = w0 + threadIdx.x; w < w1; w += kCopyThreads * kCopyUnroll) {
        uint4 v[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const long long k = w + u * kCopyThreads;
            if (k < w1) v[u] = __ldcs(from + k);
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const long long k = w + u * kCopyThreads;
            if (k < w1) __stcs(to + k, v[u]);
        }
    }
}

}  // namespace

extern "C" pa_status pa_copy_blocks(void* key_cache, void* value_cache, int num_kv_heads,
                                    int head_size, int block_size, int64_t num_blocks,
                                    pa_kv_dtype kv_dtype, const int64_t* src, const int64_t* dst,
                                    int num_pairs, uint32_t* status, void* stream) {
    g_bm_detail[0] = 0;
    if (num_pairs < 0) return bm_fail(PA_ERR_INVALID_ARG, "num_pairs < 0");
    if (num_pairs == 0) return PA_OK;
    if (!key_cache || !value_cache || !src || !dst)
        return bm_fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if ((reinterpret_cast<uintptr_t>(key_cache) | reinterpret_cast<uintptr_t>(value_cache)) % 16)
        return bm_fail(PA_ERR_INVALID_ARG, "caches must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) % 8)
        return bm_fail(PA_ERR_INVALID_ARG, "src/dst must be 8-byte aligned");
    if (status && reinterpret_cast<uintptr_t>(status) % 4)
        return bm_fail(PA_ERR_INVALID_ARG, "status must be 4-byte aligned");
    if (num_kv_heads < 1 || head_size < 1 || block_size < 1 || num_blocks < 1)
        return bm_fail(PA_ERR_INVALID_ARG, "sizes must be positive");
    if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3)
        return bm_fail(PA_ERR_UNSUPPORTED, "kv_dtype");
    const long long elem = kv_dtype == PA_KV_FP8_E4M3 ? 1 : 2;
    const long long block_bytes = static_cast<long long>(num_kv_heads) * head_size * block_size * elem;
    if (block_bytes % 16) return bm_fail(PA_ERR_UNSUPPORTED, "block bytes not a multiple of 16");
    const long long words = block_bytes / 16;
    const long long slice = kCopyThreads * kCopyUnroll * 4;  // 64 KiB per CTA
    const long long slices = (words + slice - 1) / slice;
    if (slices > 65535 || num_pairs > 0x7fffffff)
        return bm_fail(PA_ERR_UNSUPPORTED, "block too large");
    dim3 grid(static_cast<unsigned>(num_pairs), 2, static_cast<unsigned>(slices));
    pa_copy_blocks_kernel<<<grid, kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint8_t*>(key_cache), static_cast<uint8_t*>(value_cache), words, slice, src,
        dst, num_blocks, status);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return bm_fail(PA_ERR_CUDA, cudaGetErrorString(e));
    return PA_OK;
}
