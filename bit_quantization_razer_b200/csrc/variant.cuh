// Special-value set of a format variant (block size and set chosen by the
// caller for accuracy studies): up to 4 values, multiples of 0.5 in
// [2.5, 9.5], none an E2M1 magnitude.
#pragma once

namespace razer {

struct VariantV {
    float v[4];
    int nv;  // 0 (plain) .. 4
};

}  // namespace razer
