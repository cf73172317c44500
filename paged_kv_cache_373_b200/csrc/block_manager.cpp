// block_manager.cpp -- the host block manager (C ABI in
// include/pkv_block_manager.h): free list, reference counts, block tables,
// copy-on-write decisions and the prefix cache (key chain + parked LRU
// queue).  The behaviour and the readings it rests on are stated in the
// header; this file holds the data structures:
//   - free list: a FIFO of never-cached free blocks (free_order first);
//   - parked queue: an intrusive doubly linked list over block ids, least
//     recently parked at the head, O(1) removal on a cache hit;
//   - key index: hash map from a block's 32-byte key to the block;
//   - per sequence: block table, token ids, extras, keys of its full blocks.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <deque>
#include <string>
#include <unordered_map>
#include <vector>

#include "../../include/pkv_block_manager.h"
#include "pkv_internal.h"

namespace pkv {
namespace {

// ---------------------------------------------------------------------------
// SHA-256, FIPS 180-4.  The round constants and the initial hash value are
// derived here from their definition (the first 32 fractional bits of the
// cube roots of the first 64 primes, and of the square roots of the first 8)
// with exact integer roots.
// ---------------------------------------------------------------------------
using u128 = unsigned __int128;

uint64_t iroot(u128 v, int k) {  // floor(v^(1/k)) for k in {2, 3}, v < 2^110
    uint64_t lo = 0, hi = 1ull << 40;
    while (lo < hi) {
        const uint64_t mid = lo + (hi - lo + 1) / 2;
        u128 p = mid;
        for (int i = 1; i < k; ++i) p *= mid;
        if (p <= v) lo = mid; else hi = mid - 1;
    }
    return lo;
}

struct Sha256Consts {
    uint32_t k[64], h0[8];
    Sha256Consts() {
        int primes[64], n = 0;
        for (int c = 2; n < 64; ++c) {
            bool prime = true;
            for (int d = 2; d * d <= c; ++d) if (c % d == 0) { prime = false; break; }
            if (prime) primes[n++] = c;
        }
        for (int i = 0; i < 64; ++i) k[i] = (uint32_t)iroot((u128)primes[i] << 96, 3);
        for (int i = 0; i < 8; ++i) h0[i] = (uint32_t)iroot((u128)primes[i] << 64, 2);
    }
};
const Sha256Consts& sha_consts() {
    static const Sha256Consts c;
    return c;
}

inline uint32_t rotr(uint32_t x, int n) { return (x >> n) | (x << (32 - n)); }

void sha256_block(uint32_t h[8], const uint8_t* blk, const uint32_t* K) {
    uint32_t w[64];
    for (int t = 0; t < 16; ++t)
        w[t] = (uint32_t)blk[4 * t] << 24 | (uint32_t)blk[4 * t + 1] << 16 | (uint32_t)blk[4 * t + 2] << 8 |
               (uint32_t)blk[4 * t + 3];
    for (int t = 16; t < 64; ++t) {
        const uint32_t s0 = rotr(w[t - 15], 7) ^ rotr(w[t - 15], 18) ^ (w[t - 15] >> 3);
        const uint32_t s1 = rotr(w[t - 2], 17) ^ rotr(w[t - 2], 19) ^ (w[t - 2] >> 10);
        w[t] = w[t - 16] + s0 + w[t - 7] + s1;
    }
    uint32_t a = h[0], b = h[1], c = h[2], d = h[3], e = h[4], f = h[5], g = h[6], hh = h[7];
    for (int t = 0; t < 64; ++t) {
        const uint32_t S1 = rotr(e, 6) ^ rotr(e, 11) ^ rotr(e, 25);
        const uint32_t ch = (e & f) ^ (~e & g);
        const uint32_t t1 = hh + S1 + ch + K[t] + w[t];
        const uint32_t S0 = rotr(a, 2) ^ rotr(a, 13) ^ rotr(a, 22);
        const uint32_t maj = (a & b) ^ (a & c) ^ (b & c);
        const uint32_t t2 = S0 + maj;
        hh = g; g = f; f = e; e = d + t1; d = c; c = b; b = a; a = t1 + t2;
    }
    h[0] += a; h[1] += b; h[2] += c; h[3] += d; h[4] += e; h[5] += f; h[6] += g; h[7] += hh;
}

void sha256(const uint8_t* data, size_t len, uint8_t out[32]) {
    const Sha256Consts& C = sha_consts();
    uint32_t h[8];
    memcpy(h, C.h0, sizeof(h));
    size_t i = 0;
    for (; i + 64 <= len; i += 64) sha256_block(h, data + i, C.k);
    uint8_t tail[128] = {0};
    const size_t rem = len - i;
    memcpy(tail, data + i, rem);
    tail[rem] = 0x80;
    const size_t tl = rem + 1 + 8 <= 64 ? 64 : 128;
    const uint64_t bits = (uint64_t)len * 8;
    for (int j = 0; j < 8; ++j) tail[tl - 1 - j] = (uint8_t)(bits >> (8 * j));
    sha256_block(h, tail, C.k);
    if (tl == 128) sha256_block(h, tail + 64, C.k);
    for (int j = 0; j < 8; ++j) {
        out[4 * j] = (uint8_t)(h[j] >> 24); out[4 * j + 1] = (uint8_t)(h[j] >> 16);
        out[4 * j + 2] = (uint8_t)(h[j] >> 8); out[4 * j + 3] = (uint8_t)h[j];
    }
}

// ---------------------------------------------------------------------------
struct Key {
    uint8_t b[32];
    bool operator==(const Key& o) const { return memcmp(b, o.b, 32) == 0; }
};
struct KeyHash {
    size_t operator()(const Key& k) const { size_t h; memcpy(&h, k.b, sizeof h); return h; }
};

struct Seq {
    std::vector<int32_t> table;
    std::vector<int32_t> tokens;
    std::vector<Key> keys;  // keys of the full blocks, in order (prefix cache only)
    std::string extras;
};

}  // namespace
}  // namespace pkv

using namespace pkv;

struct pkv_block_manager {
    int64_t nb = 0;
    int bs = 0;
    bool cache = false;
    std::deque<int32_t> free_list;
    std::vector<int32_t> ref;
    std::vector<uint8_t> has_key;
    std::vector<Key> key_of;
    std::unordered_map<Key, int32_t, KeyHash> block_of;
    // parked LRU list: head = least recently parked; -1 terminates
    std::vector<int32_t> prev, next;
    std::vector<uint8_t> parked;
    int32_t head = -1, tail = -1;
    int64_t num_parked = 0;
    std::unordered_map<int64_t, Seq> seqs;
    int64_t next_id = 0;
    int64_t hits = 0, evictions = 0, cows = 0;

    void park(int32_t b) {
        prev[b] = tail; next[b] = -1;
        if (tail >= 0) next[tail] = b; else head = b;
        tail = b;
        parked[b] = 1;
        ++num_parked;
    }
    void unpark(int32_t b) {
        if (prev[b] >= 0) next[prev[b]] = next[b]; else head = next[b];
        if (next[b] >= 0) prev[next[b]] = prev[b]; else tail = prev[b];
        prev[b] = next[b] = -1;
        parked[b] = 0;
        --num_parked;
    }
    int64_t available() const { return (int64_t)free_list.size() + num_parked; }
    // caller has checked available() > 0
    int32_t take() {
        int32_t b;
        if (!free_list.empty()) {
            b = free_list.front();
            free_list.pop_front();
        } else {
            b = head;
            unpark(b);
            block_of.erase(key_of[b]);
            has_key[b] = 0;
            ++evictions;
        }
        ref[b] = 1;
        return b;
    }
    void drop(int32_t b) {
        if (--ref[b] == 0) {
            if (has_key[b]) park(b);
            else free_list.push_back(b);
        }
    }
    Key key_after(const Key* prev_key, const int32_t* toks, const std::string& extras) const {
        std::vector<uint8_t> buf(32 + 4 * (size_t)bs + extras.size());
        if (prev_key) memcpy(buf.data(), prev_key->b, 32);
        for (int i = 0; i < bs; ++i) {
            const uint32_t t = (uint32_t)toks[i];
            buf[32 + 4 * i] = (uint8_t)t; buf[33 + 4 * i] = (uint8_t)(t >> 8);
            buf[34 + 4 * i] = (uint8_t)(t >> 16); buf[35 + 4 * i] = (uint8_t)(t >> 24);
        }
        if (!extras.empty()) memcpy(buf.data() + 32 + 4 * bs, extras.data(), extras.size());
        Key k;
        sha256(buf.data(), buf.size(), k.b);
        return k;
    }
    void register_key(int32_t b, const Key& k) {
        if (has_key[b] || block_of.count(k)) return;  // the first holder keeps the key
        block_of.emplace(k, b);
        key_of[b] = k;
        has_key[b] = 1;
    }
    Seq* find(int64_t id) {
        auto it = seqs.find(id);
        return it == seqs.end() ? nullptr : &it->second;
    }
    const Seq* find(int64_t id) const {
        auto it = seqs.find(id);
        return it == seqs.end() ? nullptr : &it->second;
    }
    // the append of one token to s: writes slot / cow (src -1 if none)
    void append(Seq& s, int32_t token, int64_t* slot, int64_t* src, int64_t* dst) {
        const int64_t pos = (int64_t)s.tokens.size();
        const int64_t lb = pos / bs, off = pos % bs;
        *src = *dst = -1;
        if (lb == (int64_t)s.table.size()) {
            s.table.push_back(take());
        } else if (ref[s.table[lb]] > 1) {
            const int32_t old = s.table[lb];
            const int32_t nb2 = take();
            --ref[old];
            s.table[lb] = nb2;
            *src = old; *dst = nb2;
            ++cows;
        }
        s.tokens.push_back(token);
        if (cache && off == bs - 1) {  // the block just filled up
            const Key k = key_after(lb > 0 ? &s.keys[lb - 1] : nullptr, s.tokens.data() + lb * bs, s.extras);
            s.keys.push_back(k);
            register_key(s.table[lb], k);
        }
        *slot = (int64_t)s.table[lb] * bs + off;
    }
    // blocks one append to s needs, given `extra_drop[b]` copies of b already
    // taken by earlier appends of the same batch
    bool append_needs_block(const Seq& s, std::unordered_map<int32_t, int>& copied) const {
        const int64_t lb = (int64_t)s.tokens.size() / bs;
        if (lb == (int64_t)s.table.size()) return true;
        const int32_t b = s.table[lb];
        int& c = copied[b];
        if (ref[b] - c > 1) { ++c; return true; }
        return false;
    }
};

namespace {
pkv_status bm_fail(pkv_status st, const char* fmt, ...) {
    char msg[256];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(msg, sizeof msg, fmt, ap);
    va_end(ap);
    return pkv::fail(st, "%s", msg);
}
}  // namespace

extern "C" void pkv_sha256(const void* data, size_t len, uint8_t digest[32]) {
    sha256(static_cast<const uint8_t*>(data), len, digest);
}

extern "C" pkv_status pkv_bm_create(int64_t num_blocks, int block_size, const int32_t* free_order,
                                    int prefix_cache, pkv_block_manager** out) {
    if (!out) return bm_fail(PKV_EINVAL, "null out");
    *out = nullptr;
    if (num_blocks <= 0 || num_blocks > 0x7fffffffLL || block_size <= 0)
        return bm_fail(PKV_EINVAL, "num_blocks must be in [1, 2^31) and block_size positive");
    auto* bm = new pkv_block_manager;
    bm->nb = num_blocks;
    bm->bs = block_size;
    bm->cache = prefix_cache != 0;
    bm->ref.assign(num_blocks, 0);
    bm->has_key.assign(num_blocks, 0);
    bm->key_of.resize(num_blocks);
    bm->prev.assign(num_blocks, -1);
    bm->next.assign(num_blocks, -1);
    bm->parked.assign(num_blocks, 0);
    if (free_order) {
        std::vector<uint8_t> seen(num_blocks, 0);
        for (int64_t i = 0; i < num_blocks; ++i) {
            const int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete bm;
                return bm_fail(PKV_EINVAL, "free_order is not a permutation of [0, num_blocks)");
            }
            seen[b] = 1;
            bm->free_list.push_back(b);
        }
    } else {
        for (int64_t i = 0; i < num_blocks; ++i) bm->free_list.push_back((int32_t)i);
    }
    *out = bm;
    return PKV_OK;
}

extern "C" void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

extern "C" pkv_status pkv_bm_add_sequence(pkv_block_manager* bm, const int32_t* tokens, int64_t num_tokens,
                                          const void* extras, size_t extras_len, int64_t* seq_id,
                                          int64_t* cached_tokens) {
    if (!bm || !seq_id || num_tokens < 0 || (num_tokens > 0 && !tokens) || (extras_len > 0 && !extras))
        return bm_fail(PKV_EINVAL, "bad argument");
    const int bs = bm->bs;
    const int64_t nblk = (num_tokens + bs - 1) / bs, full = num_tokens / bs;
    Seq s;
    s.tokens.assign(tokens, tokens + num_tokens);
    if (extras_len) s.extras.assign(static_cast<const char*>(extras), extras_len);
    // leading run of cached full blocks
    int64_t hit = 0;
    if (bm->cache) {
        s.keys.reserve(full);
        for (int64_t i = 0; i < full; ++i)
            s.keys.push_back(bm->key_after(i ? &s.keys[i - 1] : nullptr, tokens + i * bs, s.extras));
        while (hit < full && bm->block_of.count(s.keys[hit])) ++hit;
    }
    // blocks taken from the pool: every non-hit block; a hit on a parked
    // block also removes it from the pool, so count those too
    int64_t parked_hits = 0;
    for (int64_t i = 0; i < hit; ++i) parked_hits += bm->ref[bm->block_of[s.keys[i]]] == 0;
    if (nblk - hit > bm->available() - parked_hits)
        return bm_fail(PKV_ENOBLOCKS, "prompt needs %lld blocks, %lld available",
                       (long long)(nblk - hit), (long long)(bm->available() - parked_hits));
    s.table.reserve(nblk);
    for (int64_t i = 0; i < hit; ++i) {
        const int32_t b = bm->block_of[s.keys[i]];
        if (bm->ref[b] == 0) bm->unpark(b);
        ++bm->ref[b];
        ++bm->hits;
        s.table.push_back(b);
    }
    for (int64_t i = hit; i < nblk; ++i) {
        const int32_t b = bm->take();
        if (bm->cache && i < full) bm->register_key(b, s.keys[i]);
        s.table.push_back(b);
    }
    const int64_t id = bm->next_id++;
    bm->seqs.emplace(id, std::move(s));
    *seq_id = id;
    if (cached_tokens) *cached_tokens = hit * bs;
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t* child) {
    if (!bm || !child) return bm_fail(PKV_EINVAL, "null argument");
    const Seq* p = bm->find(parent);
    if (!p) return bm_fail(PKV_EINVAL, "unknown sequence %lld", (long long)parent);
    Seq c = *p;
    for (int32_t b : c.table) ++bm->ref[b];
    const int64_t id = bm->next_id++;
    bm->seqs.emplace(id, std::move(c));
    *child = id;
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_append_token(pkv_block_manager* bm, int64_t seq_id, int32_t token, int64_t* slot,
                                          int64_t* cow_src, int64_t* cow_dst) {
    if (!bm || !slot || !cow_src || !cow_dst) return bm_fail(PKV_EINVAL, "null argument");
    Seq* s = bm->find(seq_id);
    if (!s) return bm_fail(PKV_EINVAL, "unknown sequence %lld", (long long)seq_id);
    std::unordered_map<int32_t, int> copied;
    if (bm->append_needs_block(*s, copied) && bm->available() == 0)
        return bm_fail(PKV_ENOBLOCKS, "no free block for sequence %lld", (long long)seq_id);
    bm->append(*s, token, slot, cow_src, cow_dst);
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_append_batch(pkv_block_manager* bm, const int64_t* seq_ids, const int32_t* tokens,
                                          int64_t n, int64_t* slots, int64_t* cow_pairs, int64_t* num_cow) {
    if (!bm || n < 0 || (n > 0 && (!seq_ids || !tokens || !slots || !cow_pairs)) || !num_cow)
        return bm_fail(PKV_EINVAL, "bad argument");
    std::vector<Seq*> ss(n);
    std::unordered_map<int64_t, int> seen;
    std::unordered_map<int32_t, int> copied;
    int64_t need = 0;
    for (int64_t i = 0; i < n; ++i) {
        ss[i] = bm->find(seq_ids[i]);
        if (!ss[i]) return bm_fail(PKV_EINVAL, "unknown sequence %lld", (long long)seq_ids[i]);
        if (seen[seq_ids[i]]++) return bm_fail(PKV_EINVAL, "sequence %lld twice in one batch", (long long)seq_ids[i]);
        need += bm->append_needs_block(*ss[i], copied);
    }
    if (need > bm->available())
        return bm_fail(PKV_ENOBLOCKS, "batch needs %lld blocks, %lld available", (long long)need,
                       (long long)bm->available());
    int64_t k = 0;
    for (int64_t i = 0; i < n; ++i) {
        int64_t src, dst;
        bm->append(*ss[i], tokens[i], slots + i, &src, &dst);
        if (src >= 0) { cow_pairs[2 * k] = src; cow_pairs[2 * k + 1] = dst; ++k; }
    }
    *num_cow = k;
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_free_sequence(pkv_block_manager* bm, int64_t seq_id) {
    if (!bm) return bm_fail(PKV_EINVAL, "null manager");
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return bm_fail(PKV_EINVAL, "unknown sequence %lld", (long long)seq_id);
    const std::vector<int32_t>& t = it->second.table;
    for (auto b = t.rbegin(); b != t.rend(); ++b) bm->drop(*b);  // tail parked first
    bm->seqs.erase(it);
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_seq_len(const pkv_block_manager* bm, int64_t seq_id, int64_t* len) {
    if (!bm || !len) return bm_fail(PKV_EINVAL, "null argument");
    const Seq* s = bm->find(seq_id);
    if (!s) return bm_fail(PKV_EINVAL, "unknown sequence %lld", (long long)seq_id);
    *len = (int64_t)s->tokens.size();
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_block_table(const pkv_block_manager* bm, int64_t seq_id, int32_t* table,
                                         int64_t capacity, int64_t* num_blocks) {
    if (!bm || !num_blocks || (capacity > 0 && !table)) return bm_fail(PKV_EINVAL, "null argument");
    const Seq* s = bm->find(seq_id);
    if (!s) return bm_fail(PKV_EINVAL, "unknown sequence %lld", (long long)seq_id);
    *num_blocks = (int64_t)s->table.size();
    if (capacity < *num_blocks) return bm_fail(PKV_EINVAL, "capacity %lld < %lld blocks", (long long)capacity,
                                               (long long)*num_blocks);
    std::copy(s->table.begin(), s->table.end(), table);
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_batch_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int64_t n,
                                          int32_t* tables, int64_t max_blocks_per_seq, int32_t* seq_lens) {
    if (!bm || n < 0 || max_blocks_per_seq < 0 || (n > 0 && (!seq_ids || !tables || !seq_lens)))
        return bm_fail(PKV_EINVAL, "bad argument");
    for (int64_t i = 0; i < n; ++i) {
        const Seq* s = bm->find(seq_ids[i]);
        if (!s) return bm_fail(PKV_EINVAL, "unknown sequence %lld", (long long)seq_ids[i]);
        if ((int64_t)s->table.size() > max_blocks_per_seq)
            return bm_fail(PKV_EINVAL, "sequence %lld holds %lld blocks > max_blocks_per_seq",
                           (long long)seq_ids[i], (long long)s->table.size());
    }
    for (int64_t i = 0; i < n; ++i) {
        const Seq* s = bm->find(seq_ids[i]);
        int32_t* row = tables + i * max_blocks_per_seq;
        std::copy(s->table.begin(), s->table.end(), row);
        std::fill(row + s->table.size(), row + max_blocks_per_seq, -1);
        seq_lens[i] = (int32_t)s->tokens.size();
    }
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_block_key(const pkv_block_manager* bm, int64_t seq_id, int64_t block_index,
                                       uint8_t key[32]) {
    if (!bm || !key) return bm_fail(PKV_EINVAL, "null argument");
    const Seq* s = bm->find(seq_id);
    if (!s) return bm_fail(PKV_EINVAL, "unknown sequence %lld", (long long)seq_id);
    if (!bm->cache || block_index < 0 || block_index >= (int64_t)s->keys.size())
        return bm_fail(PKV_EINVAL, "block %lld of sequence %lld has no key", (long long)block_index,
                       (long long)seq_id);
    memcpy(key, s->keys[block_index].b, 32);
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_get_stats(const pkv_block_manager* bm, pkv_bm_stats* st) {
    if (!bm || !st) return bm_fail(PKV_EINVAL, "null argument");
    pkv_bm_stats r{};
    r.num_blocks = bm->nb;
    r.block_size = bm->bs;
    r.free_blocks = (int64_t)bm->free_list.size();
    r.parked_blocks = bm->num_parked;
    r.cached_blocks = (int64_t)bm->block_of.size();
    std::vector<int32_t> fill(bm->nb, 0);
    for (const auto& kv : bm->seqs) {
        const Seq& s = kv.second;
        const int64_t n = (int64_t)s.tokens.size();
        for (size_t i = 0; i < s.table.size(); ++i) {
            const int64_t f = std::min<int64_t>(bm->bs, n - (int64_t)i * bm->bs);
            if (f > fill[s.table[i]]) fill[s.table[i]] = (int32_t)f;
        }
    }
    for (int64_t b = 0; b < bm->nb; ++b) {
        if (bm->ref[b] > 0) {
            ++r.used_blocks;
            r.token_slots += fill[b];
        }
    }
    r.reserved_slots = r.used_blocks * bm->bs;
    r.hit_blocks = bm->hits;
    r.evicted_blocks = bm->evictions;
    r.cow_copies = bm->cows;
    r.num_seqs = (int64_t)bm->seqs.size();
    *st = r;
    return PKV_OK;
}
