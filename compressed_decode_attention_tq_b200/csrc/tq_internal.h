// Host-side helpers shared by the library's translation units (not part of the ABI).
#pragma once
#include "tq.h"

namespace tqi {
// Records a message for tq_last_error() on this thread and returns st.
tq_status fail(tq_status st, const char* msg);
// Clears the per-thread message.
void clear_error();
}  // namespace tqi
