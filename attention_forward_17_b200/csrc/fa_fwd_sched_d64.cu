// Compiled schedules of the attention kernel for head dimension 64: the
// exponential split (EMU) times the K/V ring depth (SLOTS, 16 KiB a slot),
// plus the two persistent launches and the split-KV ping-pong kernel for the
// default exponential split, and the two-query-tile kernel (key tiles of 64,
// 128 and 192 rows: 2 x 192 + 2 x 64 = 512 TMEM columns; two score buffers
// per tile at 64 rows; the sum of the bf16 weights on the tensor core, whose O
// buffers are 80 columns wide).  First entry =
// default.
#include "fa_schedules.h"

namespace fa {
namespace {
const Schedule kD64[] = {
    make_schedule<64, 4, 8>(), make_schedule<64, 0, 8>(), make_schedule<64, 2, 8>(),
    make_schedule<64, 4, 4>(), make_schedule<64, 0, 4>(), make_schedule<64, 2, 4>(),
    make_schedule<64, 4, 8, 1>(), make_schedule<64, 4, 4, 1>(),
    make_schedule<64, 4, 8, 2>(), make_schedule<64, 4, 4, 2>(),
    make_pp_schedule<64, 4, 8>(), make_pp_schedule<64, 4, 4>(),
    make_pp_schedule<64, 0, 8>(),
    make_2q_schedule<64, 4, 8>(), make_2q_schedule<64, 2, 8>(), make_2q_schedule<64, 0, 8>(),
    make_2q_schedule<64, 4, 4>(),
    make_2q_schedule<64, 4, 8, 64>(), make_2q_schedule<64, 4, 8, 192>(),
    make_2q_schedule<64, 4, 8, 64, true>(),
    make_2q_schedule<64, 4, 8, 128, false, true>(),
    make_2q_schedule<64, 4, 8, 64, true, true>(), make_2q_schedule<64, 3, 8, 128, false, true>(),
    make_2q_schedule<64, 4, 8, 64, false, true, false, 3>(), make_2q_schedule<64, 2, 8, 64, false, true, false, 3>(),
    make_2q_schedule<64, 0, 8, 64, false, true, false, 3>(),
    make_2q_schedule<64, 4, 8, 80, false, true, false, 3>(), make_2q_schedule<64, 3, 8, 80, false, true, false, 3>(),
    make_2q_schedule<64, 0, 8, 80, false, true, false, 3>(),
};
}  // namespace

const Schedule* schedules_d64(int* count) {
    *count = static_cast<int>(sizeof(kD64) / sizeof(kD64[0]));
    return kD64;
}

}  // namespace fa
