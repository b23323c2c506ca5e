"""The ncu summaries under profiles/ give the commands that made them: every
such command runs committed files only, leaves the GPU clocks alone
(--clock-control none), and passes bench.py arguments that bench.py accepts."""
import glob
import os
import re
import shlex
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _commands():
    """(file, command) for every command line in the summaries: lines that
    start with `ncu ` or `python bench.py`, with backslash continuations joined."""
    out = []
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        lines = open(path, encoding="utf-8").read().splitlines()
        i = 0
        while i < len(lines):
            line = lines[i].strip()
            if line.startswith("ncu ") or line.startswith("python bench.py"):
                cmd = line
                while cmd.endswith("\\") and i + 1 < len(lines):
                    i += 1
                    cmd = cmd[:-1].rstrip() + " " + lines[i].strip()
                out.append((os.path.basename(path), cmd))
            i += 1
    return out


def _bench_parser():
    sys.path.insert(0, ROOT)
    try:
        import bench
    finally:
        sys.path.remove(ROOT)
    return bench.make_parser()


def test_every_summary_gives_its_command():
    files = {os.path.basename(p) for p in glob.glob(os.path.join(ROOT, "profiles", "*.md"))}
    with_cmd = {f for f, _ in _commands()}
    assert files and files == with_cmd, sorted(files - with_cmd)


def test_ncu_commands_keep_clocks_and_run_committed_files():
    parser = _bench_parser()
    n = 0
    for name, cmd in _commands():
        assert "/root/" not in cmd and "_work" not in cmd, (name, cmd)
        for seg in re.split(r"&&|\|\||;|\|", cmd):      # each command of a chain
            if seg.strip().startswith("ncu "):
                assert "--clock-control none" in seg, (name, cmd)
            seg = re.split(r"[<>]|\b2>", seg)[0]            # without its redirections
            words = shlex.split(seg)
            if "bench.py" in words:
                args = words[words.index("bench.py") + 1:]
                parser.parse_args(args)      # exits (SystemExit) on an unknown argument
                n += 1
    assert n > 0
