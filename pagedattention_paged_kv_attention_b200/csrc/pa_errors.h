// pa_errors.h -- makes the public header's PA_DEVERR_* bits and PA_WORKSPACE_HEADER_BYTES visible to
// the device code.
#pragma once

#include "pagedattn.h"
