// Library-internal helpers shared between the translation units of libatlaskv.
#pragma once

#include "atlaskv.h"

// Record `msg` as this thread's atlaskv_last_error() text and return `st`.
atlaskv_status akv_report(atlaskv_status st, const char *msg);
