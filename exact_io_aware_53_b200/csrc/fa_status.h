// Device error word shared by the kernels and the host API.
#pragma once

#define FA_DEV_TIMEOUT 0x1u   // a bounded wait expired
#define FA_DEV_BAD_TILE 0x2u  // a tile index fell outside the tensor (index check)

namespace fa {

// Passed by value to every kernel that waits on an mbarrier.
struct WaitCtl {
    unsigned int* status;         // device error word (FA_DEV_* bits); never null
    unsigned long long limit_ns;  // longest a single wait may take
};

}  // namespace fa
