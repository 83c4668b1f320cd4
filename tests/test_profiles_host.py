"""The ncu summaries under profiles/ state the command that produced them; every script those
commands run must be a file of this repository, and each summary must name its command."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")


def _command_blocks(text):
    return re.findall(r"```\n(.*?)```", text, flags=re.S)


def test_every_profile_names_its_command_and_runs_committed_files_only():
    names = sorted(n for n in os.listdir(PROFILES) if n.endswith((".md", ".txt")))
    assert names, "no profile summaries"
    for name in names:
        with open(os.path.join(PROFILES, name)) as f:
            text = f.read()
        commands = [b for b in _command_blocks(text) if "python" in b or "ncu" in b]
        assert commands, f"{name}: no command block"
        for block in commands:
            assert "--clock-control none" in block or "ncu" not in block, (name, block)
            for script in re.findall(r"[\w./-]+\.py\b", block):
                assert os.path.exists(os.path.join(ROOT, script)), (name, script)
                assert not script.startswith(("_work", "/")), (name, script)
