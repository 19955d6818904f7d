// status.cuh - device status flags shared by the kernels (values match the
// MOE_DEV_* flags of the public header).
#pragma once

namespace moe {
constexpr int MOE_DEV_BAD_EXPERT_ID_FLAG = 1;
constexpr int MOE_DEV_TIMEOUT_FLAG = 2;
constexpr int MOE_DEV_BAD_TABLES_FLAG = 4;
}  // namespace moe
