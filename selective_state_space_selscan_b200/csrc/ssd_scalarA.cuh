// ssd_scalarA.cuh -- scalar-A (Mamba-2 / SSD) selective scan on tcgen05.
#pragma once

namespace selscan {

constexpr int kSsdN = 128;  // state size built
constexpr int kSsdP = 64;   // head dimension built

}  // namespace selscan
