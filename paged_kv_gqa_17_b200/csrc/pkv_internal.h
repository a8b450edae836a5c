// Internal declarations shared by the host planner (pkv_host.cpp) and the
// CUDA side (pkv_decode.cu) of libpkv.so.  Not part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include "pkv.h"

namespace pkv {

constexpr int kPage = 16;          // the fast path's tokens per page
constexpr size_t kWsAlign = 256;   // workspace section alignment

// Device error word bits (pkv_workspace_status).
constexpr uint32_t kErrTimeout = 1;
constexpr uint32_t kErrSeqLen = 2;
constexpr uint32_t kErrPageId = 4;
constexpr uint32_t kErrItem = 8;

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace sections, in bytes from the workspace base.  The error word and
// the counters are zero between calls (each call leaves them so); the
// partial states need no initial value.
struct WsLayout {
    size_t error_off = 0;    // uint32 error word (+ padding)
    size_t counters_off = 0; // uint32 completion counter per (row, kv head) pair
    size_t m_off = 0;        // float m[slot][G]  (running max, log2 domain)
    size_t l_off = 0;        // float l[slot][G]
    size_t acc_off = 0;      // float acc[slot][G][D]
    size_t total = 0;
    int64_t n_slots = 0;
};

inline WsLayout ws_layout(const pkv_shape &s, const pkv_plan &p, int32_t n_items)
{
    WsLayout w;
    const int64_t pairs = (int64_t)s.B * s.H_kv;
    const int64_t G = s.H_kv > 0 ? s.H_q / s.H_kv : 0;
    if (p.mode == PKV_SPLIT_S)
        w.n_slots = pairs * p.num_splits;
    else if (p.mode == PKV_WORK_QUEUE || p.mode == PKV_BALANCED)
        w.n_slots = n_items;
    size_t off = kWsAlign;  // error word section
    w.counters_off = off;
    off += round_up((size_t)pairs * 4, kWsAlign);
    w.m_off = off;
    off += round_up((size_t)(w.n_slots * G) * 4, kWsAlign);
    w.l_off = off;
    off += round_up((size_t)(w.n_slots * G) * 4, kWsAlign);
    w.acc_off = off;
    off += round_up((size_t)(w.n_slots * G * s.head_dim) * 4, kWsAlign);
    w.total = off;
    return w;
}

// Shape checks shared by the host entry points; PKV_OK when the shape is
// well formed (fast-path support is checked separately by the decode call).
int check_shape(const pkv_shape *s);

// Balanced queue: block b owns pages [floor(b*U/T), floor((b+1)*U/T)) of
// the U pages of all (row, KV head) pairs laid end to end.
inline int64_t balanced_start(int64_t U, int64_t T, int64_t b) { return (b * U) / T; }

}  // namespace pkv
