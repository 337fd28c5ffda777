// Exception guard of the C entry points (host code only).
#pragma once

#include "kie.h"

namespace kie {

// Runs the body of a C entry point: a failed host allocation (or any other
// C++ exception) becomes KIE_ERR_HOST_MEMORY instead of crossing the C ABI.
template <class F>
kie_status no_throw(F&& body) {
  try {
    return body();
  } catch (...) {
    return KIE_ERR_HOST_MEMORY;
  }
}

}  // namespace kie
