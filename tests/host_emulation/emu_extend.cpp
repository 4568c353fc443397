// Runs the append kernel (extend_kernel: one CTA of 288 threads per (sequence, KV head)) or, with
// "mode 1", every level of the tree build (build_level_mma_kernel, one launch per level, a grid of
// at most "grid" CTAs of 512 threads striding over tiles of 128 nodes) on host threads, one
// std::thread per CUDA thread, over inputs read from a case directory, and writes the caches and
// the node arena back there.  The tensor-core steps run through host versions (emu_umma_ops.h).  Test infrastructure: it checks the kernels' barriers (every thread
// reaches each one), their memory accesses (AddressSanitizer) and their results, without a GPU.
//
// usage: emu_extend <case dir>
//   <dir>/params.txt  key value lines (scalars); "row_off", "slots", "span" lines (kMaxLevels+1
//                     ints); optional "seq_len" (one per sequence) and "pages" (the page table)
//   <dir>/{k_tok,v_tok,k_node,v_node,k_new,v_new}.bin bf16 arrays, <dir>/pooler.bin fp32 [128][128]
//   writes <dir>/{k_tok,v_tok,k_node,v_node}_out.bin
#include <cmath>
#include <fstream>
#include <memory>
#include <mutex>
#include <map>
#include <sstream>
#include <thread>

#include "extend_extracted.h"

namespace emu {
thread_local int t_tid, t_block, t_crank, t_cs, t_grid = 1;
int g_nt = 256;
thread_local float *t_tmem;
std::vector<uint32_t> g_cta_pred;
std::mutex g_mbar_mu;
std::map<const void *, std::unique_ptr<MBar>> g_mbars;
MBar &mbar_of(const void *p) {
  std::lock_guard<std::mutex> lk(g_mbar_mu);
  auto &slot = g_mbars[p];
  if (!slot) slot.reset(new MBar());
  return *slot;
}
thread_local long t_cluster_gen = -1;
thread_local unsigned char *t_smem;
std::vector<unsigned char *> g_cluster_smem;
size_t g_smem_bytes;
std::vector<TBarrier> g_cta_bar;
TBarrier g_cluster_bar;
std::vector<TBarrier> g_warp_bar;
std::vector<uint32_t> g_warp_slot;
std::vector<Where> g_where;
int g_cs = 1;

void report_and_abort(const char *why) {
  static std::mutex m;
  std::lock_guard<std::mutex> lk(m);
  fprintf(stderr, "STALL: %s\n", why);
  for (int t = 0; t < g_nt; ++t)
    fprintf(stderr, "  thread %d waits at %s:%d\n", t, (const char *)g_where[t].what, (int)g_where[t].line);
  fflush(stderr);
  _exit(3);
}
}  // namespace emu

using namespace recsa;

template <typename T>
std::vector<T> read_bin(const std::string &path) {
  std::ifstream f(path, std::ios::binary | std::ios::ate);
  if (!f) {
    fprintf(stderr, "cannot read %s\n", path.c_str());
    exit(2);
  }
  const size_t n = (size_t)f.tellg();
  std::vector<T> v(n / sizeof(T) + 1);
  f.seekg(0);
  f.read(reinterpret_cast<char *>(v.data()), (std::streamsize)n);
  v.resize(std::max<size_t>(n / sizeof(T), 1));
  return v;
}
template <typename T>
void write_bin(const std::string &path, const std::vector<T> &v) {
  std::ofstream f(path, std::ios::binary);
  f.write(reinterpret_cast<const char *>(v.data()), (std::streamsize)(v.size() * sizeof(T)));
}

template <typename Kernel>
void run_block(Kernel kernel, size_t smem_bytes, int block, int grid, int nthreads) {
  using namespace emu;
  std::vector<unsigned char> smem(smem_bytes, 0xAB);
  std::vector<float> tmem(128 * 512, std::nanf(""));
  g_nt = nthreads;
  {
    std::lock_guard<std::mutex> lk(g_mbar_mu);
    g_mbars.clear();
  }
  g_smem_bytes = smem.size();
  g_cluster_smem.assign(1, smem.data());
  g_cta_bar = std::vector<TBarrier>(1);
  g_cta_bar[0].init(nthreads, "syncthreads");
  g_cta_pred.assign(nthreads, 0u);
  g_warp_bar = std::vector<TBarrier>(nthreads / 32);
  for (auto &w : g_warp_bar) w.init(32, "warp");
  g_warp_slot.assign(nthreads, 0);
  g_where = std::vector<Where>(nthreads);
  std::vector<std::thread> th;
  for (int t = 0; t < nthreads; ++t)
    th.emplace_back([&, t] {
      t_tid = t;
      t_crank = 0;
      t_cs = 1;
      t_block = block;
      t_grid = grid;
      t_smem = smem.data();
      t_tmem = tmem.data();
      kernel();
      g_where[t].line = -1;
      g_where[t].what = "exited";
    });
  for (auto &x : th) x.join();
}

int main(int argc, char **argv) {
  if (argc != 2) {
    fprintf(stderr, "usage: emu_extend <case dir>\n");
    return 2;
  }
  const std::string dir = argv[1];
  std::map<std::string, double> kv;
  std::map<std::string, std::vector<int64_t>> lists;
  {
    std::ifstream f(dir + "/params.txt");
    std::string line;
    while (std::getline(f, line)) {
      std::istringstream ss(line);
      std::string key;
      ss >> key;
      if (key == "row_off" || key == "slots" || key == "span" || key == "seq_len" || key == "pages") {
        int64_t x;
        while (ss >> x) lists[key].push_back(x);
      } else {
        double x;
        ss >> x;
        kv[key] = x;
      }
    }
  }
  auto ktok = read_bin<uint16_t>(dir + "/k_tok.bin"), vtok = read_bin<uint16_t>(dir + "/v_tok.bin");
  auto knode = read_bin<uint16_t>(dir + "/k_node.bin"), vnode = read_bin<uint16_t>(dir + "/v_node.bin");
  auto knew = read_bin<uint16_t>(dir + "/k_new.bin"), vnew = read_bin<uint16_t>(dir + "/v_new.bin");
  auto pooler = read_bin<float>(dir + "/pooler.bin");
  std::vector<int64_t> seq_len(lists["seq_len"].begin(), lists["seq_len"].end());
  std::vector<int32_t> pages(lists["pages"].begin(), lists["pages"].end());

  ExtendArgs a = {};
  a.k_new = reinterpret_cast<const uint4 *>(knew.data());
  a.v_new = reinterpret_cast<const uint4 *>(vnew.data());
  a.k_tok = ktok.data();
  a.v_tok = vtok.data();
  a.k_node = knode.data();
  a.v_node = vnode.data();
  a.pooler = pooler.data();
  a.seq_len = seq_len.empty() ? nullptr : seq_len.data();
  const bool paged = !pages.empty();
  a.pages = paged ? pages.data() : nullptr;
  a.page_shift = (int)kv["page_shift"];
  a.num_pages = (int)kv["num_pages"];
  a.capacity = (int64_t)kv["capacity"];
  a.at = (int64_t)kv["at"];
  a.chunk = (int)kv["chunk"];
  a.hkv = (int)kv["hkv"];
  a.b = (int)kv["b"];
  a.levels = (int)kv["levels"];
  for (int l = 0; l <= kMaxLevels; ++l) {
    a.row_off[l] = lists["row_off"].at(l);
    a.slots[l] = lists["slots"].at(l);
    a.span[l] = lists["span"].at(l);
  }
  const int blocks = (int)kv["batch"] * a.hkv;
  uint32_t err_word = 0;
  a.err = &err_word;
  if ((int)kv["stuck"] == 1) {  // no product ever completes: the kernels must report and return
    emu::g_mbar_stuck = true;
    recsa::kMbarPolls = 64;
  }
  if ((int)kv["mode"] == 1) {  // the whole build, level by level, over `length` tokens
    const int64_t length = (int64_t)kv["length"];
    const int grid_cap = (int)kv["grid"];
    for (int l = 1; l <= a.levels; ++l) {
      BuildArgs g = {};
      const bool from_tokens = l == 1;
      g.src_k = from_tokens ? ktok.data() : knode.data();
      g.src_v = from_tokens ? vtok.data() : vnode.data();
      g.src_row_off = from_tokens ? 0 : a.row_off[l - 1];
      g.src_slots = a.slots[l - 1];
      g.dst_k = knode.data();
      g.dst_v = vnode.data();
      g.dst_row_off = a.row_off[l];
      g.dst_slots = a.slots[l];
      g.span_prev = a.span[l - 1];
      g.n_prev = (length + g.span_prev - 1) / g.span_prev;
      g.length = length;
      g.j0 = 0;
      g.nj = (length + a.span[l] - 1) / a.span[l];
      g.b = a.b;
      g.bh = blocks;
      g.hkv = a.hkv;
      g.span = a.span[l];
      g.seq_len = a.seq_len;
      g.pages = from_tokens ? a.pages : nullptr;
      g.page_shift = a.page_shift;
      g.pages_per_seq = paged ? a.capacity >> a.page_shift : 0;
      g.num_pages = a.num_pages;
      g.pooler = pooler.data();
      const int64_t tiles = (g.bh * g.nj + umma::kM - 1) / umma::kM;
      const int grid = (int)std::min<int64_t>(tiles, grid_cap);
      for (int blk = 0; blk < grid; ++blk) {
        if (g.pages)
          run_block([&] { build_level_mma_kernel<true>(g); }, kMmaSmem, blk, grid, kMmaThreads);
        else
          run_block([&] { build_level_mma_kernel<false>(g); }, kMmaSmem, blk, grid, kMmaThreads);
      }
    }
  } else {
    for (int blk = 0; blk < blocks; ++blk) {
      if (paged)
        run_block([&] { extend_kernel<true>(a); }, kExtendSmem, blk, blocks, kExtendThreads);
      else
        run_block([&] { extend_kernel<false>(a); }, kExtendSmem, blk, blocks, kExtendThreads);
    }
  }
  std::ofstream(dir + "/err.txt") << err_word << " " << recsa::g_build_err << "\n";
  write_bin(dir + "/k_tok_out.bin", ktok);
  write_bin(dir + "/v_tok_out.bin", vtok);
  write_bin(dir + "/k_node_out.bin", knode);
  write_bin(dir + "/v_node_out.bin", vnode);
  return 0;
}
