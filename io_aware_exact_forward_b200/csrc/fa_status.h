// fa_status.h -- status codes shared by the host and device code of libfa.
#pragma once
#include "../../include/fa.h"
