// Declarations shared between the library's translation units (not part of
// the public C ABI).
#pragma once

#include "../../include/tl.h"

__attribute__((visibility("hidden"))) tl_status tl_internal_set_error(tl_status s, const char* msg);
