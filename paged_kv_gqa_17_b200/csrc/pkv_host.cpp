// Host planner of libpkv.so: policy lookup, compact work-queue builder,
// workload counters and workspace sizing.  Pure C++, no CUDA.
//
// Sources: "PersistentKV: Page-Aware Decode Scheduling for Long-Context LLM
// Serving on Commodity GPUs" (gist.science explainer), Technical summary >
// Methodology > 1 ("Row-local bounds", "Compact work queue") and 2
// ("Calibrated adaptive policy"); Key contributions ("page-aware scheduling",
// "scheduler-induced workload counters"); Results (launch fan-out, merge-state
// traffic).
#include <algorithm>
#include <climits>
#include <cstring>
#include <unordered_set>
#include <vector>

#include "pkv_internal.h"

namespace pkv {

int check_shape(const pkv_shape *s)
{
    if (!s)
        return PKV_ERR_INVALID;
    if (s->B < 0 || s->H_q <= 0 || s->H_kv <= 0 || s->head_dim <= 0 || s->page_size <= 0)
        return PKV_ERR_INVALID;
    if (s->H_q % s->H_kv != 0 || s->max_pages_per_seq < 0 || s->num_pool_pages < 0)
        return PKV_ERR_INVALID;
    return PKV_OK;
}

namespace {

// Built-in policy table, measured on B200 by paged_kv_gqa_17_b200/calibrate.py
// (seed 20260622, checked on 20260623); generated from policy_b200.json.
const pkv_policy_rule kDefaultRules[] = {
#include "pkv_policy_table.inc"
};
constexpr int32_t kNumDefaultRules = (int32_t)(sizeof(kDefaultRules) / sizeof(kDefaultRules[0]));

int check_lens(const int32_t *lens, int32_t B)
{
    if (B > 0 && !lens)
        return PKV_ERR_INVALID;
    for (int32_t i = 0; i < B; ++i)
        if (lens[i] < 0)
            return PKV_ERR_INVALID;
    return PKV_OK;
}

int check_rules(const pkv_policy_rule *rules, int32_t n)
{
    if (n < 0 || (n > 0 && !rules))
        return PKV_ERR_INVALID;
    for (int32_t k = 0; k < n; ++k) {
        const pkv_policy_rule &r = rules[k];
        if (r.mode != PKV_NO_SPLIT && r.mode != PKV_SPLIT_S && r.mode != PKV_WORK_QUEUE && r.mode != PKV_BALANCED)
            return PKV_ERR_INVALID;
        if ((r.mode == PKV_SPLIT_S || r.mode == PKV_BALANCED) && r.num_splits < 1)
            return PKV_ERR_INVALID;
        if (r.mode == PKV_WORK_QUEUE && (r.chunk_pages < 0 || (r.chunk_pages == 0 && r.num_splits < 1)))
            return PKV_ERR_INVALID;
        if ((r.flags & PKV_FLAG_DEVICE_FILL) && (r.mode != PKV_WORK_QUEUE || r.chunk_pages != 0))
            return PKV_ERR_INVALID;
        if (r.flags & PKV_FLAG_SHARED_PREFIX)  // needs the block table: planned by the caller
            return PKV_ERR_INVALID;
    }
    return PKV_OK;
}

// Items of the compact queue at chunk size C: H_kv * sum_i max(1, ceil(pages_i / C)).
int64_t queue_items(const int32_t *lens, int32_t B, int32_t H_kv, int32_t P, int64_t C)
{
    int64_t n = 0;
    for (int32_t i = 0; i < B; ++i)
        n += std::max<int64_t>(1, ceil_div(ceil_div(lens[i], P), C));
    return n * H_kv;
}

// The smallest chunk size whose queue has at most T items (the queue fills
// one wave of T blocks with as little work per block as possible); the
// whole row (pages_max) when even one item per (row, KV head) exceeds T.
// The item count only falls as C grows, so a bisection finds it.
int64_t fill_chunk(const int32_t *lens, const pkv_shape &s, int64_t pages_max, int64_t T)
{
    if (queue_items(lens, s.B, s.H_kv, s.page_size, pages_max) > T)
        return pages_max;
    int64_t lo = 1, hi = pages_max;  // items(hi) <= T
    while (lo < hi) {
        const int64_t mid = lo + (hi - lo) / 2;
        if (queue_items(lens, s.B, s.H_kv, s.page_size, mid) <= T)
            hi = mid;
        else
            lo = mid + 1;
    }
    return lo;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" {

const char *pkv_version(void) { return "pkv-b200 0.1.0 (sm_100a)"; }

const char *pkv_status_string(int status)
{
    switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported shape or layout";
    case PKV_ERR_CAPACITY: return "buffer too small";
    case PKV_ERR_CUDA: return "CUDA error";
    case PKV_ERR_TIMEOUT: return "device wait timed out";
    case PKV_ERR_DEVICE_INPUT: return "out-of-range device input";
    default: return "unknown status";
    }
}

int pkv_default_policy(pkv_policy_rule *rules, int32_t capacity, int32_t *n_rules)
{
    if (!n_rules)
        return PKV_ERR_INVALID;
    *n_rules = kNumDefaultRules;
    if (capacity < kNumDefaultRules)
        return PKV_ERR_CAPACITY;
    if (!rules)
        return PKV_ERR_INVALID;
    std::memcpy(rules, kDefaultRules, sizeof kDefaultRules);
    return PKV_OK;
}

int pkv_select_policy(const int32_t *seq_lens_host, const pkv_shape *shape,
                      const pkv_policy_rule *rules, int32_t n_rules, pkv_plan *plan)
{
    if (!plan || check_shape(shape) != PKV_OK)
        return PKV_ERR_INVALID;
    if (!rules) {
        rules = kDefaultRules;
        n_rules = kNumDefaultRules;
    }
    int rc = check_lens(seq_lens_host, shape->B);
    if (rc == PKV_OK)
        rc = check_rules(rules, n_rules);
    if (rc != PKV_OK)
        return rc;
    const int32_t B = shape->B;
    int32_t n_max = 0;
    for (int32_t i = 0; i < B; ++i)
        n_max = std::max(n_max, seq_lens_host[i]);
    const int64_t pages_max = ceil_div(n_max, shape->page_size);
    const pkv_policy_rule *chosen = nullptr;
    for (int32_t k = 0; k < n_rules && !chosen; ++k) {
        const pkv_policy_rule &r = rules[k];
        if (r.b_lo <= B && B < r.b_hi && r.nmax_lo <= n_max && n_max < r.nmax_hi)
            chosen = &r;
    }
    if (!chosen || B == 0 || pages_max == 0) {
        *plan = {PKV_NO_SPLIT, 1, 0, 0};
        return PKV_OK;
    }
    if (chosen->mode == PKV_NO_SPLIT) {
        *plan = {PKV_NO_SPLIT, 1, 0, chosen->flags};
        return PKV_OK;
    }
    if (chosen->mode == PKV_BALANCED) {
        *plan = {PKV_BALANCED, chosen->num_splits, 0, chosen->flags};
        return PKV_OK;
    }
    if (chosen->flags & PKV_FLAG_DEVICE_FILL) {  // the chunk is found on the device, per step
        *plan = {PKV_WORK_QUEUE, chosen->num_splits, 0, chosen->flags};
        return PKV_OK;
    }
    const int64_t C = chosen->mode == PKV_SPLIT_S ? ceil_div(pages_max, chosen->num_splits)
                      : chosen->chunk_pages > 0 ? (int64_t)chosen->chunk_pages
                                                : fill_chunk(seq_lens_host, *shape, pages_max, chosen->num_splits);
    *plan = {chosen->mode, (int32_t)ceil_div(pages_max, C), (int32_t)C, chosen->flags};
    return PKV_OK;
}

int pkv_work_queue_size(const int32_t *seq_lens_host, const pkv_shape *shape, int32_t chunk_pages,
                        int32_t *n_items)
{
    if (!n_items || chunk_pages < 1 || check_shape(shape) != PKV_OK)
        return PKV_ERR_INVALID;
    int rc = check_lens(seq_lens_host, shape->B);
    if (rc != PKV_OK)
        return rc;
    const int64_t n = queue_items(seq_lens_host, shape->B, shape->H_kv, shape->page_size, chunk_pages);
    if (n > INT32_MAX)
        return PKV_ERR_CAPACITY;
    *n_items = (int32_t)n;
    return PKV_OK;
}

int pkv_build_work_queue(const int32_t *seq_lens_host, const pkv_shape *shape, int32_t chunk_pages,
                         pkv_work_item *items, int32_t capacity, int32_t *indptr, int32_t *n_items)
{
    int32_t need = 0;
    int rc = pkv_work_queue_size(seq_lens_host, shape, chunk_pages, &need);
    if (rc != PKV_OK)
        return rc;
    *n_items = need;
    if (capacity < need)
        return PKV_ERR_CAPACITY;
    if ((need > 0 && !items) || !indptr)
        return PKV_ERR_INVALID;
    const int64_t span = (int64_t)chunk_pages * shape->page_size;
    int32_t k = 0;
    for (int32_t i = 0; i < shape->B; ++i) {
        const int32_t n = seq_lens_host[i];
        for (int32_t h = 0; h < shape->H_kv; ++h) {
            indptr[(int64_t)i * shape->H_kv + h] = k;
            if (n == 0) {
                items[k++] = {i, h, 0, 0};
                continue;
            }
            for (int64_t b = 0; b < n; b += span)
                items[k++] = {i, h, (int32_t)b, (int32_t)std::min<int64_t>(b + span, n)};
        }
    }
    indptr[(int64_t)shape->B * shape->H_kv] = k;
    return PKV_OK;
}

}  // extern "C"

namespace pkv {
namespace {

// Walks the balanced queue of a batch; calls emit(row, kv_head, tok_begin,
// tok_end, block) for every item in order.  Returns the item count.
template <typename Emit>
int64_t walk_balanced(const int32_t *lens, const pkv_shape &s, int32_t T, Emit emit)
{
    const int64_t P = s.page_size;
    int64_t U = 0;
    for (int32_t i = 0; i < s.B; ++i)
        U += ceil_div(lens[i], P);
    U *= s.H_kv;
    // last block whose share starts at or before page u
    auto owner = [&](int64_t u, int64_t hint) {
        int64_t b = hint;
        while (b + 1 < T && balanced_start(U, T, b + 1) <= u)
            ++b;
        return b;
    };
    int64_t n = 0, u = 0, b = 0;
    for (int32_t i = 0; i < s.B; ++i) {
        const int64_t N = lens[i];
        const int64_t pg = ceil_div(N, P);
        for (int32_t h = 0; h < s.H_kv; ++h) {
            if (N == 0) {
                b = owner(u, b);
                emit(i, h, 0, 0, b);
                ++n;
            }
            for (int64_t x = u; x < u + pg;) {
                b = owner(x, b);
                const int64_t y = std::min(u + pg, balanced_start(U, T, b + 1));
                emit(i, h, (x - u) * P, std::min((y - u) * P, N), b);
                ++n;
                x = y;
            }
            u += pg;
        }
    }
    return n;
}

}  // namespace
}  // namespace pkv

extern "C" {

int pkv_balanced_queue_size(const int32_t *seq_lens_host, const pkv_shape *shape, int32_t n_blocks,
                            int32_t *n_items)
{
    if (!n_items || n_blocks < 1 || check_shape(shape) != PKV_OK)
        return PKV_ERR_INVALID;
    int rc = check_lens(seq_lens_host, shape->B);
    if (rc != PKV_OK)
        return rc;
    const int64_t n = walk_balanced(seq_lens_host, *shape, n_blocks, [](int32_t, int32_t, int64_t, int64_t, int64_t) {});
    if (n > INT32_MAX)
        return PKV_ERR_CAPACITY;
    *n_items = (int32_t)n;
    return PKV_OK;
}

int pkv_fill_queue_capacity(const pkv_shape *shape, int32_t n_blocks, int32_t *capacity)
{
    if (!capacity || n_blocks < 1 || check_shape(shape) != PKV_OK)
        return PKV_ERR_INVALID;
    // at most T items, or one per (row, KV head) when whole rows exceed T
    const int64_t c = std::max<int64_t>(n_blocks, (int64_t)shape->B * shape->H_kv);
    if (c > INT32_MAX)
        return PKV_ERR_CAPACITY;
    *capacity = (int32_t)c;
    return PKV_OK;
}

int pkv_balanced_queue_capacity(const pkv_shape *shape, int32_t n_blocks, int32_t *capacity)
{
    if (!capacity || n_blocks < 1 || check_shape(shape) != PKV_OK)
        return PKV_ERR_INVALID;
    // each item is one pair's run inside one share: at most one per pair plus one
    // per share boundary falling inside a pair's pages (T - 1 of them)
    const int64_t c = (int64_t)shape->B * shape->H_kv + n_blocks;
    if (c > INT32_MAX)
        return PKV_ERR_CAPACITY;
    *capacity = (int32_t)c;
    return PKV_OK;
}

int pkv_build_balanced_queue(const int32_t *seq_lens_host, const pkv_shape *shape, int32_t n_blocks,
                             pkv_work_item *items, int32_t capacity, int32_t *indptr, int32_t *n_items)
{
    int32_t need = 0;
    int rc = pkv_balanced_queue_size(seq_lens_host, shape, n_blocks, &need);
    if (rc != PKV_OK)
        return rc;
    *n_items = need;
    if (capacity < need)
        return PKV_ERR_CAPACITY;
    if ((need > 0 && !items) || !indptr)
        return PKV_ERR_INVALID;
    const int64_t pairs = (int64_t)shape->B * shape->H_kv;
    int32_t *pair_ptr = indptr;
    int32_t *block_ptr = indptr + pairs + 1;
    int32_t k = 0;
    int64_t last_pair = -1, next_block = 0;
    walk_balanced(seq_lens_host, *shape, n_blocks, [&](int32_t i, int32_t h, int64_t tb, int64_t te, int64_t b) {
        const int64_t pair = (int64_t)i * shape->H_kv + h;
        while (last_pair < pair)
            pair_ptr[++last_pair] = k;
        while (next_block <= b)
            block_ptr[next_block++] = k;
        items[k++] = {i, h, (int32_t)tb, (int32_t)te};
    });
    while (last_pair < pairs)
        pair_ptr[++last_pair] = k;
    while (next_block <= n_blocks)
        block_ptr[next_block++] = k;
    return PKV_OK;
}

int pkv_plan_counters(const int32_t *seq_lens_host, const pkv_shape *shape, const pkv_plan *plan,
                      pkv_counters *c)
{
    if (!plan || !c || check_shape(shape) != PKV_OK)
        return PKV_ERR_INVALID;
    int rc = check_lens(seq_lens_host, shape->B);
    if (rc != PKV_OK)
        return rc;
    const int64_t B = shape->B, H_kv = shape->H_kv, D = shape->head_dim, P = shape->page_size;
    const int64_t G = shape->H_q / shape->H_kv;
    const int64_t state = G * (D + 2) * 4;
    const int64_t S = plan->num_splits, C = plan->chunk_pages;
    const bool separate = (plan->flags & PKV_FLAG_SEPARATE_MERGE) != 0;
    pkv_counters out{};
    int64_t zero_rows = 0, tokens = 0, pages = 0;
    std::unordered_set<int32_t> distinct;
    for (int64_t i = 0; i < B; ++i) {
        const int32_t n = seq_lens_host[i];
        zero_rows += n == 0;
        tokens += n;
        pages += ceil_div(n, P);
        if (n > 0)
            distinct.insert(n);
    }
    switch (plan->mode) {
    case PKV_NO_SPLIT:
        out.launches = 1;
        out.work_items = B * H_kv;
        out.empty_items = H_kv * zero_rows;
        break;
    case PKV_SPLIT_S: {
        if (S < 1 || C < 1)
            return PKV_ERR_INVALID;
        out.launches = 1 + separate;
        out.work_items = B * H_kv * S;
        int64_t empty = 0;
        for (int64_t i = 0; i < B; ++i)
            empty += S - std::min<int64_t>(S, ceil_div(ceil_div(seq_lens_host[i], P), C));
        out.empty_items = H_kv * empty;
        out.merge_state_bytes = S > 1 ? 2 * B * H_kv * S * state : 0;
        break;
    }
    case PKV_WORK_QUEUE: {
        if (plan->flags & PKV_FLAG_SHARED_PREFIX)  // the units depend on the block table
            return PKV_ERR_UNSUPPORTED;
        const bool device_fill = (plan->flags & PKV_FLAG_DEVICE_FILL) != 0;
        int64_t Cq = C;
        if (device_fill) {  // the chunk the blocks find on the device for these lengths
            if (S < 1 || C != 0)
                return PKV_ERR_INVALID;
            int64_t pages_max = 0;
            for (int64_t i = 0; i < B; ++i)
                pages_max = std::max<int64_t>(pages_max, ceil_div(seq_lens_host[i], P));
            Cq = pages_max == 0 ? 1 : fill_chunk(seq_lens_host, *shape, pages_max, S);
        }
        if (Cq < 1)
            return PKV_ERR_INVALID;
        out.launches = 1 + separate;
        int64_t items = 0, multi = 0;
        for (int64_t i = 0; i < B; ++i) {
            const int64_t k = std::max<int64_t>(1, ceil_div(ceil_div(seq_lens_host[i], P), Cq));
            items += k;
            if (k > 1)
                multi += k;
        }
        out.work_items = H_kv * items;
        out.empty_items = H_kv * zero_rows;
        out.merge_state_bytes = 2 * H_kv * multi * state;
        out.queue_bytes = device_fill ? 0 : 16 * out.work_items + 4 * (B * H_kv + 1);
        break;
    }
    case PKV_BALANCED: {
        if (S < 1)
            return PKV_ERR_INVALID;
        out.launches = 1 + separate;
        out.work_items = S;
        out.empty_items = H_kv * zero_rows;
        std::vector<int32_t> per_pair((size_t)(B * H_kv), 0);
        const int64_t n = walk_balanced(seq_lens_host, *shape, (int32_t)S,
                                        [&](int32_t i, int32_t h, int64_t, int64_t, int64_t) {
                                            ++per_pair[(size_t)((int64_t)i * H_kv + h)];
                                        });
        int64_t multi = 0;
        for (int32_t k : per_pair)
            if (k > 1)
                multi += k;
        out.merge_state_bytes = 2 * multi * state;
        out.queue_bytes = 16 * n + 4 * (B * H_kv + 1) + 4 * (S + 1);
        break;
    }
    default:
        return PKV_ERR_INVALID;
    }
    out.kv_bytes = tokens * H_kv * 2 * D * 2;
    out.kv_bytes_streamed = pages * P * H_kv * 2 * D * 2;
    out.q_bytes = B * shape->H_q * D * 2;
    out.out_bytes = out.q_bytes;
    out.bucket_launches = 2 * (int64_t)distinct.size();
    *c = out;
    return PKV_OK;
}

int pkv_workspace_bytes(const pkv_shape *shape, const pkv_plan *plan, int32_t n_items, size_t *bytes)
{
    if (!plan || !bytes || check_shape(shape) != PKV_OK || n_items < 0)
        return PKV_ERR_INVALID;
    if (plan->mode == PKV_SPLIT_S && plan->num_splits < 1)
        return PKV_ERR_INVALID;
    *bytes = ws_layout(*shape, *plan, n_items).total;
    return PKV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Prefix-sharing work queue ["Chapter 8 - Next-generation KV cache management"
// (actionbridge.io), 8.1 reference-counted block sharing and 8.3 prefix
// caches: rows whose block tables start with the same physical pages; PKV,
// Methodology 1 "Compact work queue", "Row-local bounds"].

namespace pkv {
namespace {

// Sharing groups of a batch: rows with at least one full page grouped by
// their first physical page (the lowest row leads); a group's shared length
// is the number of leading table entries every member has in common with
// the leader, counting only pages that are full in every member.  Groups of
// one row, or with no shared page, are dropped.  group_of[i] = the group of
// row i or -1; shared[g] = its length in pages; rows[g] = its rows, ascending.
struct PrefixGroups {
    std::vector<int32_t> group_of;
    std::vector<int64_t> shared;
    std::vector<std::vector<int32_t>> rows;
};

PrefixGroups prefix_groups(const int32_t *lens, const int32_t *bt, const pkv_shape &s)
{
    const int64_t P = s.page_size, W = s.max_pages_per_seq;
    PrefixGroups g;
    g.group_of.assign((size_t)s.B, -1);
    std::vector<std::pair<int32_t, int32_t>> firsts;  // (first page, row) of rows with a full page
    for (int32_t i = 0; i < s.B; ++i)
        if (lens[i] >= P && W > 0)
            firsts.push_back({bt[(int64_t)i * W], i});
    std::stable_sort(firsts.begin(), firsts.end(),
                     [](const std::pair<int32_t, int32_t> &a, const std::pair<int32_t, int32_t> &b) {
                         return a.first < b.first;
                     });
    std::vector<std::vector<int32_t>> cand;
    for (size_t k = 0; k < firsts.size();) {
        size_t e = k;
        std::vector<int32_t> rows;
        while (e < firsts.size() && firsts[e].first == firsts[k].first)
            rows.push_back(firsts[e++].second);
        if (rows.size() >= 2)
            cand.push_back(rows);  // rows ascending (stable sort of ascending rows)
        k = e;
    }
    // groups in the order of their leading row
    std::sort(cand.begin(), cand.end(),
              [](const std::vector<int32_t> &a, const std::vector<int32_t> &b) { return a[0] < b[0]; });
    for (const std::vector<int32_t> &rows : cand) {
        const int32_t lead = rows[0];
        int64_t L = std::min<int64_t>(lens[lead] / P, W);
        for (size_t m = 1; m < rows.size(); ++m) {
            const int64_t full = std::min<int64_t>(lens[rows[m]] / P, W);
            int64_t k = 0;
            while (k < std::min(full, L) && bt[(int64_t)rows[m] * W + k] == bt[(int64_t)lead * W + k])
                ++k;
            L = std::min(L, k);
        }
        if (L < 1)
            continue;
        for (int32_t r : rows)
            g.group_of[(size_t)r] = (int32_t)g.rows.size();
        g.shared.push_back(L);
        g.rows.push_back(rows);
    }
    return g;
}

// Walks the prefix-sharing queue: item counts per (row, head) and, for a
// grouped row, how many of its first items are shared chunks.
int64_t prefix_row_items(int64_t n, int64_t L, int64_t span, int64_t P, int64_t *shared_chunks)
{
    if (n == 0) {
        *shared_chunks = 0;
        return 1;
    }
    const int64_t sc = ceil_div(L * P, span);
    *shared_chunks = sc;
    return sc + ceil_div(n - L * P, span);
}

}  // namespace
}  // namespace pkv

extern "C" {

int pkv_prefix_queue_size(const int32_t *seq_lens_host, const int32_t *block_table_host, const pkv_shape *shape,
                          int32_t chunk_pages, int32_t max_members, int32_t *n_items, int32_t *n_units)
{
    if (!n_items || !n_units || chunk_pages < 1 || max_members < 1 || check_shape(shape) != PKV_OK)
        return PKV_ERR_INVALID;
    int rc = check_lens(seq_lens_host, shape->B);
    if (rc != PKV_OK)
        return rc;
    if (shape->B > 0 && shape->max_pages_per_seq > 0 && !block_table_host)
        return PKV_ERR_INVALID;
    for (int32_t i = 0; i < shape->B; ++i)
        if ((int64_t)seq_lens_host[i] > (int64_t)shape->max_pages_per_seq * shape->page_size)
            return PKV_ERR_INVALID;
    const PrefixGroups g = prefix_groups(seq_lens_host, block_table_host, *shape);
    const int64_t P = shape->page_size, span = (int64_t)chunk_pages * P;
    int64_t items = 0, merged = 0;
    for (int32_t i = 0; i < shape->B; ++i) {
        const int32_t gi = g.group_of[(size_t)i];
        int64_t sc = 0;
        items += shape->H_kv * prefix_row_items(seq_lens_host[i], gi >= 0 ? g.shared[(size_t)gi] : 0, span, P, &sc);
    }
    for (size_t k = 0; k < g.rows.size(); ++k) {
        const int64_t m = (int64_t)g.rows[k].size();
        merged += shape->H_kv * ceil_div(g.shared[k] * P, span) * (m - ceil_div(m, max_members));
    }
    if (items > INT32_MAX)
        return PKV_ERR_CAPACITY;
    *n_items = (int32_t)items;
    *n_units = (int32_t)(items - merged);
    return PKV_OK;
}

int pkv_build_prefix_queue(const int32_t *seq_lens_host, const int32_t *block_table_host, const pkv_shape *shape,
                           int32_t chunk_pages, int32_t max_members, pkv_work_item *items, int32_t capacity,
                           int32_t *indptr, int32_t indptr_capacity, int32_t *n_items, int32_t *n_units)
{
    int32_t need = 0, units = 0;
    int rc = pkv_prefix_queue_size(seq_lens_host, block_table_host, shape, chunk_pages, max_members, &need, &units);
    if (rc != PKV_OK)
        return rc;
    *n_items = need;
    *n_units = units;
    const int64_t pairs = (int64_t)shape->B * shape->H_kv;
    if (capacity < need || (int64_t)indptr_capacity < pairs + 1 + units + 1 + need)
        return PKV_ERR_CAPACITY;
    if ((need > 0 && !items) || !indptr)
        return PKV_ERR_INVALID;
    const PrefixGroups g = prefix_groups(seq_lens_host, block_table_host, *shape);
    const int64_t P = shape->page_size, span = (int64_t)chunk_pages * P, H_kv = shape->H_kv;
    std::vector<int32_t> pos((size_t)shape->B, 0);  // a grouped row's place in its group
    for (const std::vector<int32_t> &rows : g.rows)
        for (size_t k = 0; k < rows.size(); ++k)
            pos[(size_t)rows[k]] = (int32_t)k;
    int32_t k = 0;
    for (int32_t i = 0; i < shape->B; ++i) {
        const int64_t n = seq_lens_host[i];
        const int32_t gi = g.group_of[(size_t)i];
        const int64_t L = gi >= 0 ? g.shared[(size_t)gi] : 0;
        for (int32_t h = 0; h < shape->H_kv; ++h) {
            indptr[(int64_t)i * H_kv + h] = k;
            if (n == 0) {
                items[k++] = {i, h, 0, 0};
                continue;
            }
            for (int64_t b = 0; b < L * P; b += span)
                items[k++] = {i, h, (int32_t)b, (int32_t)std::min<int64_t>(b + span, L * P)};
            for (int64_t b = L * P; b < n; b += span)
                items[k++] = {i, h, (int32_t)b, (int32_t)std::min<int64_t>(b + span, n)};
        }
    }
    indptr[pairs] = k;
    // units in the order of their first member: walking the items in order, a
    // shared chunk opens its run's unit when its row starts a run of
    // max_members rows of the group; other shared chunks ride in that unit
    int32_t *unit_ptr = indptr + pairs + 1;
    int32_t *unit_items = unit_ptr + units + 1;
    int32_t u = 0, m = 0;
    for (int32_t x = 0; x < k; ++x) {
        const pkv_work_item &it = items[x];
        const int32_t gi = g.group_of[(size_t)it.row];
        const int64_t c = x - indptr[(int64_t)it.row * H_kv + it.kv_head];
        const bool shared_chunk = gi >= 0 && it.tok_end > it.tok_begin && it.tok_begin < g.shared[(size_t)gi] * P;
        if (!shared_chunk) {
            unit_ptr[u++] = m;
            unit_items[m++] = x;
            continue;
        }
        const std::vector<int32_t> &rows = g.rows[(size_t)gi];
        const int32_t p = pos[(size_t)it.row];
        if (p % max_members != 0)
            continue;  // rides in the unit its run's first row opened
        unit_ptr[u++] = m;
        for (int32_t q = p; q < (int32_t)rows.size() && q < p + max_members; ++q)
            unit_items[m++] = indptr[(int64_t)rows[(size_t)q] * H_kv + it.kv_head] + (int32_t)c;
    }
    unit_ptr[u] = m;
    return PKV_OK;
}

}  // extern "C"
