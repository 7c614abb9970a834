/* NVTX 3 injection client used by the tests: records every range push (with
 * its name) and pop that the process makes, so that a test can check which
 * NVTX ranges a library call opened and that each was closed.
 *
 * NVTX loads this library from the path in NVTX_INJECTION64_PATH on the
 * process's first NVTX call and calls InitializeInjectionNvtx2, which points
 * the core module's RangePushA and RangePop slots at the recorders below.
 * Build: gcc -shared -fPIC -I<cuda>/include nvtx_recorder.c -o libnvtx_recorder.so
 */
#include <stdio.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#define REC_CAP 8192
#define REC_LEN 80

static char rec_log[REC_CAP][REC_LEN];
static int rec_n;
static int rec_depth;
static int rec_overflow;

static void rec_put(char kind, const char* name) {
  if (rec_n >= REC_CAP) {
    rec_overflow = 1;
    return;
  }
  snprintf(rec_log[rec_n], REC_LEN, "%c%s", kind, name ? name : "");
  ++rec_n;
}

/* RangePushA returns the zero-based nesting level of the range it opens. */
static int NVTX_API rec_push(const char* message) {
  rec_put('+', message);
  return rec_depth++;
}

/* RangePop returns the level of the range it closes, or a negative value
 * when no range is open. */
static int NVTX_API rec_pop(void) {
  rec_put('-', "");
  return --rec_depth;
}

int NVTX_API InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
  const NvtxExportTableCallbacks* cb =
      (const NvtxExportTableCallbacks*)get_table(NVTX_ETID_CALLBACKS);
  NvtxFunctionTable table = 0;
  unsigned int size = 0;
  if (cb == 0 || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &size) || table == 0)
    return 0;
  if (size < NVTX_CBID_CORE_RangePop) return 0;
  *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)rec_push;
  *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)rec_pop;
  return 1;
}

int nvtx_recorder_count(void) { return rec_n; }
int nvtx_recorder_overflow(void) { return rec_overflow; }
int nvtx_recorder_depth(void) { return rec_depth; }
const char* nvtx_recorder_entry(int i) { return (i >= 0 && i < rec_n) ? rec_log[i] : ""; }
void nvtx_recorder_clear(void) { rec_n = 0; rec_overflow = 0; }
