// Compiled schedules of the attention kernel for head dimension 128: the
// exponential split (EMU) times the K/V ring depth (SLOTS), every combination
// that fits 227 KiB of shared memory (a slot is one 32 KiB K or V tile, the Q
// tile takes another 32 KiB, so at most five slots; at least four keep the
// ring's parity waits sound), plus the two persistent launches and the split-KV ping-pong kernel (P in shared
// memory, which leaves room for a four-slot ring only) (one CTA per SM
// walking several query tiles) for the default exponential split, and the
// two-query-tile kernel (Q_0 and Q_1 take 64 KiB, so at most five 128-row
// slots; its ring is sound at any depth) over the exponential split and with
// 64-row key tiles (two score and two output buffers of 2 x 192 + 2 x 128
// columns would not fit TMEM, so no 192-row tiles at this head dimension).  First entry =
// default.
#include "fa_schedules.h"

namespace fa {
namespace {
const Schedule kD128[] = {
    make_schedule<128, 4, 5>(), make_schedule<128, 0, 5>(), make_schedule<128, 2, 5>(),
    make_schedule<128, 4, 4>(), make_schedule<128, 0, 4>(), make_schedule<128, 2, 4>(),
    make_schedule<128, 4, 5, 1>(), make_schedule<128, 4, 4, 1>(),
    make_schedule<128, 4, 5, 2>(), make_schedule<128, 4, 4, 2>(),
    make_pp_schedule<128, 4, 4>(), make_pp_schedule<128, 0, 4>(),
    make_2q_schedule<128, 4, 5>(), make_2q_schedule<128, 8, 5>(), make_2q_schedule<128, 2, 5>(),
    make_2q_schedule<128, 0, 5>(), make_2q_schedule<128, 4, 3>(), make_2q_schedule<128, 3, 5>(),
    make_2q_schedule<128, 4, 8, 64>(),
    make_2q_schedule<128, 4, 8, 64, true>(), make_2q_schedule<128, 0, 8, 64, true>(),
    make_2q_schedule<128, 4, 5, 128, false, false, true>(), make_2q_schedule<128, 3, 5, 128, false, false, true>(),
    make_2q_schedule<128, 0, 5, 128, false, false, true>(),
};
}  // namespace

const Schedule* schedules_d128(int* count) {
    *count = static_cast<int>(sizeof(kD128) / sizeof(kD128[0]));
    return kD128;
}

}  // namespace fa
