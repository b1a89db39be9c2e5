// Schedule table of the attention kernel: for each head dimension, masking
// mode and sequence-length bucket (N <= n_max), the exponential split, the
// K/V ring depth, the causal launch group, the launch form, the algorithm and
// the key-tile rows.  Written by
// attention_forward_17_b200/schedule_search.py on NVIDIA B200 (2026-12-03).
#pragma once

#include <cstdint>

namespace fa {

struct ScheduleTableEntry {
    int d;
    int causal;
    int64_t n_max;
    int emu;
    int slots;
    int group;
    int persist;
    int alg;
    int bn;
};

constexpr ScheduleTableEntry kScheduleTable[] = {
    {128, 0, 2048, 4, 5, 1, 0, 2, 128},
    {128, 0, 8192, 0, 5, 1, 0, 6, 128},
    {128, 0, INT64_MAX, 0, 5, 1, 0, 6, 128},
    {128, 1, 2048, 3, 5, 16, 0, 2, 128},
    {128, 1, 8192, 0, 5, 16, 0, 6, 128},
    {128, 1, INT64_MAX, 0, 5, 4, 0, 6, 128},
    {64, 0, 2048, 4, 8, 1, 0, 4, 128},
    {64, 0, 8192, 4, 8, 1, 0, 12, 64},
    {64, 0, INT64_MAX, 3, 8, 1, 0, 12, 80},
    {64, 1, 2048, 4, 8, 16, 0, 5, 64},
    {64, 1, 8192, 4, 8, 16, 0, 12, 80},
    {64, 1, INT64_MAX, 4, 8, 16, 0, 12, 80},
};

}  // namespace fa
